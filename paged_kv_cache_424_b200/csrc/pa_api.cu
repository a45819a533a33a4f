// pa_api.cu -- the extern "C" entry points declared in include/pa.h: host-side
// argument validation, the split-KV plan, and dispatch to the launchers.
#include <cstdarg>
#include <cstdint>
#include <cmath>
#include <cstdio>

#include "../../include/pa.h"
#include "pa_common.cuh"
#include "pa_decode.h"

namespace {

thread_local char g_err[512] = "";

pa_status fail(pa_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return st;
}

pa_status cuda_fail(cudaError_t e, const char *what) {
    return fail(PA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Automatic partition size, measured on B200: 512 tokens for the CUDA-core
// kernel (its per-warp rings favour many short items); for the tensor-core
// kernel at least 1024 tokens (8 chunks of 128), whose per-CTA set-up
// (TMEM, barriers, Q tile) then amortises over more chunks, and more for
// batches large enough (tc_auto_partition).  The merge costs ~1-2% of the
// KV traffic either way.
constexpr int kAutoPartitionSimt = 512;
constexpr int kAutoPartitionTc = 1024;
constexpr int kMaxPartitionTokens = 32768;

bool kv_fp8(const pa_dims *d) { return d->kv_dtype == PA_FP8_E4M3; }
int32_t kv_elem_bytes(const pa_dims *d) { return kv_fp8(d) ? 1 : 2; }

// Checks of the fields every call uses.  `attention` adds the query-side ones.
pa_status check_dims(const pa_dims *d, bool attention) {
    if (!d) return fail(PA_ERR_NULL, "dims is NULL");
    if (d->dtype != PA_F16 && d->dtype != PA_BF16) return fail(PA_ERR_DTYPE, "dtype %d is not PA_F16/PA_BF16", d->dtype);
    if (d->kv_dtype != 0 && d->kv_dtype != d->dtype && d->kv_dtype != PA_FP8_E4M3)
        return fail(PA_ERR_DTYPE, "kv_dtype %d: must be 0, dtype (%d) or PA_FP8_E4M3", d->kv_dtype, d->dtype);
    if (d->num_kv_heads <= 0 || d->head_dim <= 0 || d->block_size <= 0 || d->num_blocks <= 0)
        return fail(PA_ERR_SHAPE, "num_kv_heads, head_dim, block_size and num_blocks must be positive");
    if (d->block_size != 16) return fail(PA_ERR_UNSUPPORTED, "block_size %d: only 16 is built", d->block_size);
    if (d->head_dim != 64 && d->head_dim != 128)
        return fail(PA_ERR_UNSUPPORTED, "head_dim %d: only 64 and 128 are built", d->head_dim);
    if (!attention) return PA_OK;
    if (d->num_seqs < 0 || d->num_heads <= 0 || d->max_blocks_per_seq < 0)
        return fail(PA_ERR_SHAPE, "num_seqs and max_blocks_per_seq must be >= 0, num_heads > 0");
    if (d->num_seqs > 65535 || d->num_heads > 65535)
        return fail(PA_ERR_SHAPE, "num_seqs and num_heads must be <= 65535 (grid limits)");
    if (d->num_heads % d->num_kv_heads != 0)
        return fail(PA_ERR_SHAPE, "num_heads %d is not a multiple of num_kv_heads %d", d->num_heads, d->num_kv_heads);
    const int g = d->num_heads / d->num_kv_heads;
    if (g != 1 && g != 2 && g != 4 && g != 8 && g != 16)
        return fail(PA_ERR_UNSUPPORTED, "group size %d: only 1, 2, 4, 8, 16 are built", g);
    return PA_OK;
}

struct Plan {
    int part_blocks = 1;
    int max_parts = 1;
    size_t o_bytes = 0;    // partial outputs
    size_t lse_off = 0;    // offset of the lse array
    size_t ws_bytes = 0;   // total workspace (0 when unsplit)
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Rows per KV head (group x query tokens) rounded up to a built capacity.
int row_capacity(int rows) {
    int c = 1;
    while (c < rows) c <<= 1;
    return c;
}

// Row capacity of the tensor-core kernel for these dims, or 0 for the
// CUDA-core kernel: GQA groups (and multi-token queries) of 4 rows or more
// at head_dim 128, where the CUDA-core kernel turns ALU-bound, for 16-bit
// and FP8 caches alike.  With 1 or 2 rows the CUDA-core kernel is faster
// (measured on B200: over an FP8 cache 122 us against 273 us for the 7B MHA
// batch, whose rows would pad the MMA's 16 columns).
int tc_rows(const pa_dims *d, int rows) {
    return pa::decode_tc_supported(d->head_dim, rows, d->num_blocks, d->num_kv_heads) ? rows : 0;
}

// Multiprocessors of the current device (148 on B200 if it does not answer).
int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
        return n;
    cudaGetLastError();
    return 148;
}

// Resident tensor-core CTAs on the device: 2 per SM with 16 rows or the
// wide FP8 shape, 3 otherwise.
int64_t tc_slots(int rows, bool fp8) { return (int64_t)sm_count() * (rows > 8 || (fp8 && rows >= 8) ? 2 : 3); }

// Tokens one tensor-core CTA streams at most when it groups partitions:
// 2048 over 16-bit caches, 4096 over FP8 ones, whose chunks take half the
// time and so pay relatively twice the per-CTA cost (measured at the 70B
// shape's 512-token partitions: 184.4 us grouped to 2048 against 188.8 at
// 1024; over FP8 116.3 us grouped to 4096).
int tc_group_blocks(bool fp8) { return fp8 ? 256 : 128; }

// Partitions one tensor-core CTA streams back to back: partitions shorter
// than the group size that start on a chunk are grouped up to it per CTA,
// which saves the per-CTA set-up (TMEM, barriers, Q tile, pipeline fill and
// drain; measured: the 70B shape at 512-token partitions ran at 0.78 of the
// copy roofline against 0.87 at 1024), as long as the grid keeps at least
// two waves of resident CTAs.  The CTA writes one partial for the group, in
// its first partition's slot, and marks the others empty for the merge.
int tc_parts_per_cta(const Plan &pl, int num_seqs, int num_kv_heads, int rows, bool fp8) {
    const int group = tc_group_blocks(fp8);
    if (pl.max_parts <= 1 || pl.part_blocks % 8 != 0 || pl.part_blocks >= group) return 1;
    const int64_t slots = tc_slots(rows, fp8);
    const int64_t pairs = (int64_t)num_seqs * num_kv_heads;
    int ppc = group / pl.part_blocks;
    while (ppc > 1 && pairs * ((pl.max_parts + ppc - 1) / ppc) < 2 * slots) ppc >>= 1;
    return ppc;
}

// KV heads one tensor-core CTA streams back to back (plain decode only: the
// query rows of two heads of a group of 4 or 8 fit the Q tile's 16 rows).
// Short sequences give CTAs of a few chunks, each paying the set-up and the
// first loads' latency (measured: 1 chunk per CTA ran at 0.72 of the
// throughput of 8); two heads per CTA halve that count.  Only with
// 1024-token partitions or a single one (a CTA then streams at most 16
// chunks) and while the grid keeps two waves of resident CTAs.
int tc_heads_per_cta(const Plan &pl, const pa_dims *d, int rows, bool plain) {
    if (!plain || (pl.max_parts > 1 && pl.part_blocks < 64) || pl.part_blocks > 64) return 1;
    const int64_t slots = (int64_t)sm_count() * 3;
    int hpc = 1;
    if (2 * rows <= 16 && d->num_kv_heads % 2 == 0 && (int64_t)d->num_seqs * (d->num_kv_heads / 2) >= 2 * slots)
        hpc = 2;
    return hpc;
}

// Automatic partition of the tensor-core kernel: the largest of 4096 (FP8
// caches, and the 16-row shape that runs two CTAs per SM), 2048 and 1024
// tokens at which the batch still gives two waves of resident CTAs.  A CTA
// pays its set-up, first loads and drain once per partition.  Measured: the
// 8B continuous-batching step 156 us at 2048 against 159 at 1024 and 173 at
// 4096 over a 16-bit cache, 102 us at 4096, 109 at 2048 and 141 at 1024
// over an FP8 one; the 8B step with 4 query tokens (16 rows) 260.6 us at
// 4096 against 267.0 at 2048.
int tc_auto_partition(const pa_dims *d, int ctx_blocks, int rows, bool fp8) {
    const int64_t pairs = (int64_t)d->num_seqs * d->num_kv_heads;
    const bool wide = fp8 || rows > 8;
    for (int P = wide ? 4 * kAutoPartitionTc : 2 * kAutoPartitionTc; P > kAutoPartitionTc; P /= 2) {
        const int blocks = P / 16;
        if (pairs * ((ctx_blocks + blocks - 1) / blocks) >= 2 * tc_slots(rows, fp8)) return P;
    }
    return kAutoPartitionTc;
}

pa_status make_plan(const pa_dims *d, int32_t max_context_len, int32_t partition_tokens, Plan *pl,
                    int32_t q_len = 1, int32_t window = 0) {
    if (max_context_len < 0) return fail(PA_ERR_SHAPE, "max_context_len %d < 0", max_context_len);
    if ((int64_t)max_context_len > (int64_t)d->max_blocks_per_seq * d->block_size)
        return fail(PA_ERR_SHAPE, "max_context_len %d exceeds max_blocks_per_seq * block_size = %lld", max_context_len,
                    (long long)d->max_blocks_per_seq * d->block_size);
    if (partition_tokens < 0 || partition_tokens % 16 != 0 || partition_tokens > kMaxPartitionTokens)
        return fail(PA_ERR_SHAPE, "partition_tokens %d must be 0 or a positive multiple of 16 up to %d",
                    partition_tokens, kMaxPartitionTokens);
    const int g = d->num_heads / d->num_kv_heads;
    const int rows = tc_rows(d, row_capacity(g * q_len));
    int ctx_blocks = (max_context_len + 15) / 16;
    if (window > 0) {
        // attended positions of a sequence span at most window + q_len - 1
        // tokens, which may straddle one more block boundary
        const int64_t span_blocks = ((int64_t)window + q_len - 1 + 15) / 16 + 1;
        if (span_blocks < ctx_blocks) ctx_blocks = (int)span_blocks;
    }
    const int P = partition_tokens != 0 ? partition_tokens
                  : rows                ? tc_auto_partition(d, ctx_blocks, rows, kv_fp8(d))
                                        : kAutoPartitionSimt;
    int part_blocks = P / 16;
    const int max_parts = ctx_blocks == 0 ? 1 : (ctx_blocks + part_blocks - 1) / part_blocks;
    if (max_parts == 1) part_blocks = ctx_blocks > 0 ? ctx_blocks : 1;  // one partition: size it to the context
    pl->part_blocks = part_blocks;
    pl->max_parts = max_parts;
    if (max_parts > 1) {
        const size_t wrows = (size_t)d->num_seqs * q_len * d->num_heads * max_parts;
        pl->o_bytes = align_up(wrows * d->head_dim * sizeof(float), 256);
        pl->lse_off = pl->o_bytes;
        pl->ws_bytes = pl->o_bytes + align_up(wrows * sizeof(float), 256);
    }
    return PA_OK;
}

// Shared body of pa_decode and pa_decode_fp8 (dims already checked).  For a
// 16-bit cache k_scale = v_scale = 1.
pa_status decode_impl(void *out, const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *block_tables, const int32_t *context_lens, float scale, float k_scale,
                      float v_scale, int32_t num_kv_heads, const pa_dims *dims, int32_t max_context_len,
                      int32_t partition_tokens, void *workspace, size_t workspace_bytes, void *stream,
                      int32_t q_len = 1, int32_t window = 0, const int32_t *seq_order = nullptr) {
    pa_status st;
    if (num_kv_heads != dims->num_kv_heads)
        return fail(PA_ERR_SHAPE, "num_kv_heads %d != dims->num_kv_heads %d", num_kv_heads, dims->num_kv_heads);
    Plan pl;
    st = make_plan(dims, max_context_len, partition_tokens, &pl, q_len, window);
    if (st != PA_OK) return st;
    if (dims->num_seqs == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !context_lens || (!block_tables && dims->max_blocks_per_seq > 0))
        return fail(PA_ERR_NULL, "a required pointer is NULL");
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
        return fail(PA_ERR_ALIGN, "out, q, k_cache and v_cache must be 16-byte aligned");
    if (pl.ws_bytes > 0) {
        if (!workspace || workspace_bytes < pl.ws_bytes)
            return fail(PA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", pl.ws_bytes,
                        workspace ? workspace_bytes : (size_t)0);
        if (!aligned16(workspace)) return fail(PA_ERR_ALIGN, "workspace must be 16-byte aligned");
    }
    pa::DecodeParams p{};
    p.out = out;
    p.q = q;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.scale_log2 = scale * 1.4426950408889634f * k_scale;
    p.v_scale = v_scale;
    p.num_seqs = dims->num_seqs;
    p.num_heads = dims->num_heads;
    p.num_kv_heads = dims->num_kv_heads;
    p.max_blocks_per_seq = dims->max_blocks_per_seq;
    p.num_blocks = dims->num_blocks;
    p.part_blocks = pl.part_blocks;
    p.max_parts = pl.max_parts;
    p.ws_o = pl.ws_bytes ? static_cast<float *>(workspace) : nullptr;
    p.ws_lse = pl.ws_bytes ? reinterpret_cast<float *>(static_cast<char *>(workspace) + pl.lse_off) : nullptr;
    const int g = dims->num_heads / dims->num_kv_heads;
    p.group = g;
    p.q_len = q_len;
    p.window = window;
    p.seq_order = seq_order;
    const int rows = row_capacity(g * q_len);
    const int tc = tc_rows(dims, rows);
    const bool fp8 = kv_fp8(dims);
    p.parts_per_cta = tc ? tc_parts_per_cta(pl, dims->num_seqs, dims->num_kv_heads, tc, fp8) : 1;
    // the plain tensor-core variant: one query token, no window, unscaled 16-bit V
    const bool plain = tc && !fp8 && q_len == 1 && window == 0 && v_scale == 1.f;
    p.heads_per_cta = plain && p.parts_per_cta == 1 ? tc_heads_per_cta(pl, dims, tc, true) : 1;
    // Over an FP8 cache the tensor-core grid launches every sequence's first
    // partition before any later one: the CTAs of partitions past short
    // sequences (which read the context length and leave) then come in the
    // second half of the launch instead of between the busy ones (measured
    // on the 8B continuous-batching step: 116.7 -> 107.5 us; the 16-bit
    // shapes lost 1-2 % with it and keep the sequence-major order).
    const int64_t part_groups = (pl.max_parts + p.parts_per_cta - 1) / p.parts_per_cta;
    p.part_major = tc && fp8 && part_groups <= 65535 ? 1 : 0;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaError_t e = tc ? pa::launch_decode_tc(p, dims->dtype, tc, fp8, cs)
                       : pa::launch_decode_partitioned(p, dims->dtype, dims->head_dim, rows, fp8, cs);
    if (e != cudaSuccess) return cuda_fail(e, fp8 ? "pa_decode_fp8 launch" : "pa_decode launch");
    return PA_OK;
}

pa_status check_opts(const pa_dims *d, const pa_decode_opts *o) {
    if (!o) return fail(PA_ERR_NULL, "opts is NULL");
    if (o->q_len < 1 || o->window < 0) return fail(PA_ERR_SHAPE, "q_len %d must be >= 1, window %d >= 0", o->q_len,
                                                  o->window);
    if (!(o->k_scale > 0.f) || !(o->v_scale > 0.f) || !isfinite(o->k_scale) || !isfinite(o->v_scale))
        return fail(PA_ERR_SHAPE, "k_scale and v_scale must be finite and positive");
    const int64_t rows = (int64_t)(d->num_heads / d->num_kv_heads) * o->q_len;
    if (rows > 16) return fail(PA_ERR_UNSUPPORTED, "group * q_len = %lld: at most 16 query rows per KV head",
                               (long long)rows);
    return PA_OK;
}

}  // namespace

namespace pa {
// Lets other entry points of the library report through pa_last_error().
pa_status set_last_error(pa_status st, const char *msg) { return fail(st, "%s", msg); }
}  // namespace pa

extern "C" {

const char *pa_last_error(void) { return g_err; }

int32_t pa_version(void) { return 100; }

size_t pa_decode_workspace_size(const pa_dims *dims, int32_t max_context_len, int32_t partition_tokens) {
    if (check_dims(dims, true) != PA_OK) return (size_t)-1;
    Plan pl;
    if (make_plan(dims, max_context_len, partition_tokens, &pl) != PA_OK) return (size_t)-1;
    return pl.ws_bytes;
}

int32_t pa_decode_num_partitions(const pa_dims *dims, int32_t max_context_len, int32_t partition_tokens) {
    pa_status st = check_dims(dims, true);
    if (st != PA_OK) return st;
    Plan pl;
    st = make_plan(dims, max_context_len, partition_tokens, &pl);
    if (st != PA_OK) return st;
    return pl.max_parts;
}

pa_status pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                    const int32_t *context_lens, float scale, int32_t num_kv_heads, const pa_dims *dims,
                    int32_t max_context_len, int32_t partition_tokens, void *workspace, size_t workspace_bytes,
                    void *stream) {
    pa_status st = check_dims(dims, true);
    if (st != PA_OK) return st;
    if (kv_fp8(dims)) return fail(PA_ERR_DTYPE, "pa_decode: kv_dtype is PA_FP8_E4M3, call pa_decode_fp8");
    return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, scale, 1.f, 1.f, num_kv_heads, dims,
                       max_context_len, partition_tokens, workspace, workspace_bytes, stream);
}

pa_status pa_decode_fp8(void *out, const void *q, const void *k_cache, const void *v_cache,
                        const int32_t *block_tables, const int32_t *context_lens, float scale, float k_scale,
                        float v_scale, int32_t num_kv_heads, const pa_dims *dims, int32_t max_context_len,
                        int32_t partition_tokens, void *workspace, size_t workspace_bytes, void *stream) {
    pa_status st = check_dims(dims, true);
    if (st != PA_OK) return st;
    if (!kv_fp8(dims)) return fail(PA_ERR_DTYPE, "pa_decode_fp8: dims->kv_dtype must be PA_FP8_E4M3");
    if (!(k_scale > 0.f) || !(v_scale > 0.f) || !isfinite(k_scale) || !isfinite(v_scale))
        return fail(PA_ERR_SHAPE, "k_scale and v_scale must be finite and positive");
    return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, scale, k_scale, v_scale, num_kv_heads,
                       dims, max_context_len, partition_tokens, workspace, workspace_bytes, stream);
}

size_t pa_decode_ext_workspace_size(const pa_dims *dims, const pa_decode_opts *opts, int32_t max_context_len,
                                    int32_t partition_tokens) {
    if (check_dims(dims, true) != PA_OK || check_opts(dims, opts) != PA_OK) return (size_t)-1;
    Plan pl;
    if (make_plan(dims, max_context_len, partition_tokens, &pl, opts->q_len, opts->window) != PA_OK)
        return (size_t)-1;
    return pl.ws_bytes;
}

pa_status pa_decode_ext(void *out, const void *q, const void *k_cache, const void *v_cache,
                        const int32_t *block_tables, const int32_t *context_lens, float scale, int32_t num_kv_heads,
                        const pa_dims *dims, const pa_decode_opts *opts, int32_t max_context_len,
                        int32_t partition_tokens, void *workspace, size_t workspace_bytes, void *stream) {
    pa_status st = check_dims(dims, true);
    if (st != PA_OK) return st;
    st = check_opts(dims, opts);
    if (st != PA_OK) return st;
    return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, scale, opts->k_scale, opts->v_scale,
                       num_kv_heads, dims, max_context_len, partition_tokens, workspace, workspace_bytes, stream,
                       opts->q_len, opts->window, opts->seq_order);
}

pa_status pa_reshape_and_cache(const void *key, const void *value, void *k_cache, void *v_cache,
                               const int64_t *slot_mapping, int32_t num_tokens, const pa_dims *dims, void *stream) {
    pa_status st = check_dims(dims, false);
    if (st != PA_OK) return st;
    if (num_tokens < 0) return fail(PA_ERR_SHAPE, "num_tokens %d < 0", num_tokens);
    if (num_tokens == 0) return PA_OK;
    if (!key || !value || !k_cache || !v_cache || !slot_mapping) return fail(PA_ERR_NULL, "a required pointer is NULL");
    if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache))
        return fail(PA_ERR_ALIGN, "key, value and caches must be 16-byte aligned");
    if (kv_fp8(dims)) return fail(PA_ERR_DTYPE, "pa_reshape_and_cache: kv_dtype is PA_FP8_E4M3, call pa_reshape_and_cache_fp8");
    pa::CacheDims cd{dims->num_kv_heads, dims->head_dim, dims->num_blocks, 2};
    cudaError_t e = pa::launch_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, num_tokens, cd,
                                                 static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "pa_reshape_and_cache launch");
    return PA_OK;
}

pa_status pa_reshape_and_cache_fp8(const void *key, const void *value, void *k_cache, void *v_cache,
                                   const int64_t *slot_mapping, int32_t num_tokens, const pa_dims *dims,
                                   float k_scale, float v_scale, void *stream) {
    pa_status st = check_dims(dims, false);
    if (st != PA_OK) return st;
    if (!kv_fp8(dims)) return fail(PA_ERR_DTYPE, "pa_reshape_and_cache_fp8: dims->kv_dtype must be PA_FP8_E4M3");
    if (!(k_scale > 0.f) || !(v_scale > 0.f) || !isfinite(k_scale) || !isfinite(v_scale))
        return fail(PA_ERR_SHAPE, "k_scale and v_scale must be finite and positive");
    if (num_tokens < 0) return fail(PA_ERR_SHAPE, "num_tokens %d < 0", num_tokens);
    if (num_tokens == 0) return PA_OK;
    if (!key || !value || !k_cache || !v_cache || !slot_mapping) return fail(PA_ERR_NULL, "a required pointer is NULL");
    if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache))
        return fail(PA_ERR_ALIGN, "key, value and caches must be 16-byte aligned");
    pa::CacheDims cd{dims->num_kv_heads, dims->head_dim, dims->num_blocks, 1};
    cudaError_t e = pa::launch_reshape_and_cache_fp8(key, value, k_cache, v_cache, slot_mapping, num_tokens, cd,
                                                     dims->dtype, k_scale, v_scale, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "pa_reshape_and_cache_fp8 launch");
    return PA_OK;
}

pa_status pa_copy_blocks(void *const *k_caches, void *const *v_caches, int32_t num_layers,
                         const int64_t *block_mapping, int32_t num_pairs, const pa_dims *dims, void *stream) {
    pa_status st = check_dims(dims, false);
    if (st != PA_OK) return st;
    if (num_layers < 0 || num_pairs < 0) return fail(PA_ERR_SHAPE, "num_layers and num_pairs must be >= 0");
    if (num_layers == 0 || num_pairs == 0) return PA_OK;
    if (!k_caches || !v_caches || !block_mapping) return fail(PA_ERR_NULL, "a required pointer is NULL");
    for (int i = 0; i < num_layers; ++i) {
        if (!k_caches[i] || !v_caches[i]) return fail(PA_ERR_NULL, "cache pointer of layer %d is NULL", i);
        if (!aligned16(k_caches[i]) || !aligned16(v_caches[i]))
            return fail(PA_ERR_ALIGN, "cache pointers of layer %d must be 16-byte aligned", i);
    }
    if (num_pairs > 65535) return fail(PA_ERR_SHAPE, "num_pairs %d > 65535", num_pairs);
    pa::CacheDims cd{dims->num_kv_heads, dims->head_dim, dims->num_blocks, kv_elem_bytes(dims)};
    cudaError_t e = pa::launch_copy_blocks(k_caches, v_caches, num_layers, block_mapping, num_pairs, cd,
                                           static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "pa_copy_blocks launch");
    return PA_OK;
}

// The address the device uses for `p`: itself for device / managed memory,
// the mapped address for page-locked host memory; nullptr when the device
// cannot address it (pageable host memory).
const void *device_address(const void *p) {
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) return p;
    if (a.type == cudaMemoryTypeHost) return a.devicePointer;
    return nullptr;
}

pa_status pa_swap_blocks(const void *src_k, const void *src_v, int64_t src_num_blocks, void *dst_k, void *dst_v,
                         int64_t dst_num_blocks, const int64_t *block_mapping, int32_t num_pairs, const pa_dims *dims,
                         void *stream) {
    pa_status st = check_dims(dims, false);
    if (st != PA_OK) return st;
    if (num_pairs < 0 || src_num_blocks <= 0 || dst_num_blocks <= 0)
        return fail(PA_ERR_SHAPE, "num_pairs must be >= 0 and both pools must have blocks");
    if (num_pairs == 0) return PA_OK;
    if (num_pairs > 65535) return fail(PA_ERR_SHAPE, "num_pairs %d > 65535", num_pairs);
    if (!src_k || !src_v || !dst_k || !dst_v || !block_mapping) return fail(PA_ERR_NULL, "a required pointer is NULL");
    if (!aligned16(src_k) || !aligned16(src_v) || !aligned16(dst_k) || !aligned16(dst_v))
        return fail(PA_ERR_ALIGN, "pools must be 16-byte aligned");
    const void *sk = device_address(src_k), *sv = device_address(src_v);
    const void *dk = device_address(dst_k), *dv = device_address(dst_v);
    const void *bm = device_address(block_mapping);
    if (!sk || !sv || !dk || !dv || !bm)
        return fail(PA_ERR_MEMORY, "a pool or the mapping is not device or page-locked host memory");
    pa::CacheDims cd{dims->num_kv_heads, dims->head_dim, dims->num_blocks, kv_elem_bytes(dims)};
    cudaError_t e = pa::launch_swap_blocks(sk, sv, src_num_blocks, const_cast<void *>(dk), const_cast<void *>(dv),
                                           dst_num_blocks, static_cast<const int64_t *>(bm), num_pairs, cd,
                                           static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "pa_swap_blocks launch");
    return PA_OK;
}

pa_status pa_check_wait_timeout(int32_t milliseconds, void *stream) {
    if (milliseconds < 1 || milliseconds > 2000)
        return fail(PA_ERR_SHAPE, "milliseconds %d must be in [1, 2000]", milliseconds);
    int dev = 0, khz = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev);
    if (e != cudaSuccess || khz <= 0) return cuda_fail(e != cudaSuccess ? e : cudaErrorInvalidValue, "clock rate");
    e = pa::launch_wait_timeout_probe((long long)khz * milliseconds, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "pa_check_wait_timeout launch");
    return PA_OK;
}

pa_status pa_device_error(void *stream, uint32_t *word) {
    if (!word) return fail(PA_ERR_NULL, "word is NULL");
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "pa_device_error sync");
    unsigned int w = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&w, pa::g_device_error, sizeof w);
    if (e != cudaSuccess) return cuda_fail(e, "pa_device_error read");
    e = cudaMemcpyToSymbol(pa::g_device_error, &zero, sizeof zero);
    if (e != cudaSuccess) return cuda_fail(e, "pa_device_error clear");
    *word = w;
    return PA_OK;
}

}  // extern "C"
