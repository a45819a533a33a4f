/*
 * pa.h -- C ABI of the paged decode attention library (libpa.so, sm_100a).
 *
 * The operations of one decode step of one attention layer over a KV cache
 * stored in fixed 16-token physical blocks, and their variants:
 *
 *   pa_reshape_and_cache  write each new token's key/value into its slot
 *   pa_copy_blocks        copy-on-write duplication of shared blocks
 *   pa_swap_blocks        block copies between device and host pools (preemption)
 *   pa_decode_fp8, pa_reshape_and_cache_fp8   the same over FP8 E4M3 caches
 *   pa_decode_ext         several query tokens per sequence and/or a sliding
 *                         window, over a 16-bit or FP8 cache
 *   pa_prefix_cache_*, pa_prefix_order   host prefix cache (block-hash
 *                         lookup) and the shared-prefix-aware decode order
 *   pa_decode             single-query attention of every sequence over its
 *                         cached tokens, gathered through its block table
 *
 * Sources: "vLLM PagedAttention 大模型推理架构深度实战" (ybb.press) section 2.2
 * (16-token blocks, per-sequence block table mapping logical to physical
 * blocks), section 2.3 (copy-on-write of a block whose reference count is
 * above one), section 5.1 (exact attention combined by online softmax) and
 * section 六 (decode loop: read the KV cache, attend, write the new token's
 * K/V into its block); "vLLM：重塑大模型推理性能的关键引擎" (unionyoga.cn),
 * PagedAttention section, kernel sketch (ceil(context_len / BLOCK_SIZE)
 * blocks per sequence, table row stride MAX_BLOCKS).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every data pointer is a DEVICE pointer on the current CUDA device,
 *   except: the two pointer ARRAYS of pa_copy_blocks (host memory holding
 *   device pointers); the pools of pa_swap_blocks (device or page-locked
 *   host memory); and the arrays of pa_prefix_cache_* and pa_prefix_order
 *   (host memory).  The caller owns every buffer.
 * - The library allocates nothing and never synchronises the stream: work
 *   is enqueued on `stream` (a cudaStream_t passed as void*; NULL is the
 *   legacy default stream) and the call returns.
 * - Element type of q, out, key and value: 16-bit, fp16 or bf16
 *   (pa_dims.dtype); caches hold the same type or FP8 E4M3 codes
 *   (pa_dims.kv_dtype).  Arithmetic is fp32; outputs round to nearest-even.
 * - Layouts (row-major, contiguous):
 *     q, out         [num_seqs, num_heads, head_dim] ([num_seqs, q_len,
 *                    num_heads, head_dim] for pa_decode_ext)
 *     k/v cache      [num_blocks, num_kv_heads, block_size, head_dim]
 *     block_tables   int32 [num_seqs, max_blocks_per_seq]
 *     context_lens   int32 [num_seqs]
 *     key, value     [num_tokens, num_kv_heads, head_dim]
 *     slot_mapping   int64 [num_tokens]; slot = block * block_size + offset
 *     block_mapping  int64 [num_pairs, 2]; (src block, dst block)
 * - Query head h reads KV head h / (num_heads / num_kv_heads).
 * - Supported: block_size 16, head_dim 64 or 128, num_heads / num_kv_heads
 *   in {1, 2, 4, 8, 16}.  Data pointers must be 16-byte aligned.
 * - Host-side argument errors return a negative pa_status before anything
 *   is enqueued; pa_last_error() then describes the problem.
 * - Device data (table entries, lengths, slots) is range-checked inside the
 *   kernels: an out-of-range value is never dereferenced; it is replaced by
 *   a safe value or skipped, and a bit is set in a device error word that
 *   pa_device_error() returns.
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pa_status {
    PA_OK = 0,
    PA_ERR_NULL = -1,        /* a required pointer is NULL */
    PA_ERR_DTYPE = -2,       /* dtype is not PA_F16 / PA_BF16 */
    PA_ERR_SHAPE = -3,       /* inconsistent or negative sizes */
    PA_ERR_UNSUPPORTED = -4, /* block_size / head_dim / group size not built */
    PA_ERR_WORKSPACE = -5,   /* workspace missing or smaller than required */
    PA_ERR_CUDA = -6,        /* a CUDA launch or query failed */
    PA_ERR_ALIGN = -7,       /* a data pointer is not 16-byte aligned */
    PA_ERR_MEMORY = -8       /* a pointer the device cannot address (pageable host memory) */
} pa_status;

typedef enum pa_dtype {
    PA_F16 = 0,
    PA_BF16 = 1,
    PA_FP8_E4M3 = 2 /* KV caches only: OCP FP8 E4M3 codes, one fp32 scale per tensor */
} pa_dtype;

/* Bits of the device error word (pa_device_error). */
#define PA_DEVERR_BLOCK_ID 1u    /* a block-table entry outside [0, num_blocks) */
#define PA_DEVERR_CONTEXT 2u     /* context_len < 0, above max_blocks_per_seq*16,
                                    or above the max_context_len given */
#define PA_DEVERR_SLOT 4u        /* a slot_mapping entry beyond the pool */
#define PA_DEVERR_COPY_PAIR 8u   /* a block_mapping id outside [0, num_blocks) */
#define PA_DEVERR_TIMEOUT 16u    /* a pipeline wait gave up (bounded spin) */
#define PA_DEVERR_LAYOUT 32u     /* internal shared-memory alignment check failed */

typedef struct pa_dims {
    int32_t num_seqs;           /* S: sequences in the batch */
    int32_t num_heads;          /* H: query heads */
    int32_t num_kv_heads;       /* Hk: KV heads (H % Hk == 0) */
    int32_t head_dim;           /* D: 64 or 128 */
    int32_t block_size;         /* B: tokens per block, 16 */
    int32_t max_blocks_per_seq; /* MB: row stride of block_tables */
    int64_t num_blocks;         /* NB: physical blocks in each cache */
    int32_t dtype;              /* pa_dtype of q, out, key, value (PA_F16 / PA_BF16) */
    int32_t kv_dtype;           /* pa_dtype of the K / V caches; 0 (= PA_F16) or the value of
                                   dtype means "same as dtype", PA_FP8_E4M3 an FP8 cache */
} pa_dims;

/*
 * Bytes of device workspace pa_decode needs for these dims, the largest
 * context length it will see and the partition size (0 = automatic; else a
 * positive multiple of 16 tokens).  0 means no workspace is needed (every
 * sequence fits in one partition).  Returns (size_t)-1 for invalid dims.
 */
size_t pa_decode_workspace_size(const pa_dims *dims, int32_t max_context_len,
                                int32_t partition_tokens);

/*
 * Number of KV partitions per sequence pa_decode will use (1 = unsplit),
 * or a negative pa_status for invalid arguments.
 */
int32_t pa_decode_num_partitions(const pa_dims *dims, int32_t max_context_len,
                                 int32_t partition_tokens);

/*
 * Decode attention (ybb.press section 2.2 + 5.1; unionyoga.cn kernel sketch).
 * For every sequence s and query head h, with n = context_lens[s] and
 * K_s[j] = k_cache[block_tables[s, j / 16], h / (H / Hk), j % 16, :]:
 *     out[s, h, :] = sum_{j < n} softmax_j(scale * q[s, h, :] . K_s[j]) V_s[j]
 * A sequence with n == 0 gets an all-zero row.  Only the first
 * ceil(n / 16) table entries and the first n slots are read.
 *
 * num_kv_heads must equal dims->num_kv_heads (it is the pages' explicit
 * argument; the duplicate guards against a caller mixing layers).
 * max_context_len is a host-known upper bound on context_lens (it sizes the
 * partition grid); lengths above it are clamped and flagged.
 * partition_tokens: 0 = automatic (the CUDA-core kernel: 512 tokens; the
 * tensor-core kernel: the largest of 4096 (FP8 caches and 16 query rows
 * per KV head only), 2048 and 1024
 * tokens at which num_seqs x num_kv_heads x ceil(max_context_len / P) still
 * reaches two waves of resident CTAs), else a positive multiple of 16; with
 * more than one
 * partition, partial results go to `workspace` (at least
 * pa_decode_workspace_size() bytes, 256-byte aligned, contents ignored on
 * entry) and a log-sum-exp merge kernel combines them.
 * Enqueues one or two kernels on `stream`.
 */
pa_status pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *block_tables, const int32_t *context_lens, float scale,
                    int32_t num_kv_heads, const pa_dims *dims, int32_t max_context_len,
                    int32_t partition_tokens, void *workspace, size_t workspace_bytes,
                    void *stream);

/*
 * pa_decode_noalloc -- pa_decode for callers that cannot allocate device
 * memory.  The paper has no counterpart: this is a library convenience.
 *
 * Some callers have no way to hand pa_decode a workspace: a serving engine
 * that has already given nearly all of HBM to its KV-cache pool and forbids
 * further allocations, a plugin running inside a host framework whose memory
 * pool it may not touch, or code on a path where cudaMalloc's implicit
 * device synchronisation is not acceptable.  This entry point takes the same
 * arguments as pa_decode minus the workspace and uses instead a scratch
 * array that the library itself holds in device memory: 64 MiB
 * (67108864 bytes), reserved on every GPU that loads the library until the
 * process exits.
 *
 * - A call whose split-KV plan needs more than 64 MiB (see
 *   pa_decode_workspace_size) returns PA_ERR_WORKSPACE with a message and
 *   enqueues nothing; use pa_decode, larger partitions or fewer sequences.
 * - It allocates nothing: no cudaMalloc, no cudaFree, no allocating library.
 * - The first call on each device that needs scratch looks up the array's
 *   device address (cudaGetSymbolAddress, with that device current) and
 *   keeps it; make that first call before any stream capture.
 * - All calls on a device share the one array, which keeps the last call's
 *   contents.  Nothing in it needs to start at zero (each call writes every
 *   partial result it later reads), but calls whose kernels overlap on the
 *   GPU (different streams, or several host threads) race on it: order them
 *   on one stream or use pa_decode with separate workspaces.
 * - If a pipeline wait gives up (PA_DEVERR_TIMEOUT in pa_device_error), the
 *   output of that call is undefined: the merge may have read partial
 *   results an earlier call left in the shared array.
 * Results are those of pa_decode with the same arguments.
 */
pa_status pa_decode_noalloc(void *out, const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *block_tables, const int32_t *context_lens, float scale,
                            int32_t num_kv_heads, const pa_dims *dims, int32_t max_context_len,
                            int32_t partition_tokens, void *stream);

/*
 * Decode attention over FP8 E4M3 caches (dims->kv_dtype == PA_FP8_E4M3), a
 * variant of pa_decode that reads half the bytes.  The pages name FP8 for
 * weights ("vLLM PagedAttention 大模型推理架构深度实战" section 5.2) and
 * KV-cache compression as a goal (section 九 item 3).  Same definition as
 * pa_decode with K_s[j] = decode(k code) * k_scale and V_s[j] = decode(v code)
 * * v_scale; q / out in dims->dtype.  With 4, 8 or 16 query rows per KV
 * head (the group, or group x query tokens through pa_decode_ext) at
 * head_dim 128 the tensor cores multiply the E4M3 codes as stored: q is
 * split into three E4M3 parts under a power-of-two factor per row (q
 * recovered to within 2^-15 of the row's largest |q|, for any finite q,
 * fp16 or bf16) and the softmax weights w into four (|error| <= 2^-12 w +
 * 2^-22).  Other shapes run on the CUDA-core kernel, which widens each code
 * exactly.  Workspace as from pa_decode_workspace_size with the same dims.
 */
pa_status pa_decode_fp8(void *out, const void *q, const void *k_cache, const void *v_cache,
                        const int32_t *block_tables, const int32_t *context_lens, float scale,
                        float k_scale, float v_scale, int32_t num_kv_heads, const pa_dims *dims,
                        int32_t max_context_len, int32_t partition_tokens, void *workspace,
                        size_t workspace_bytes, void *stream);

/*
 * Cache write into FP8 E4M3 caches: for every token t with slot >= 0 and KV
 * head h, each element of key[t, h, :] (dims->dtype) becomes the E4M3 code
 * nearest to float(x) / k_scale (one correctly rounded fp32 division; ties to
 * the even code; magnitudes beyond 448 clamp to 448; NaN stays NaN); the same
 * for value with v_scale.  One kernel on `stream`.
 */
pa_status pa_reshape_and_cache_fp8(const void *key, const void *value, void *k_cache, void *v_cache,
                                   const int64_t *slot_mapping, int32_t num_tokens, const pa_dims *dims,
                                   float k_scale, float v_scale, void *stream);

/*
 * Options of pa_decode_ext.  q_len query tokens per sequence (speculative
 * verification: "vLLM PagedAttention 大模型推理架构深度实战" section 九 item 2),
 * a sliding window (the same page, section 7.2, recommends it for long
 * contexts) and per-tensor scales of the cached elements.
 */
typedef struct pa_decode_opts {
    int32_t q_len;  /* >= 1; group * q_len <= 16 (group = num_heads / num_kv_heads) */
    int32_t window; /* >= 0 tokens; 0 = no window */
    float k_scale;  /* K element = stored value * k_scale; finite, > 0 (1 for a plain cache) */
    float v_scale;  /* V element = stored value * v_scale; finite, > 0 */
    const int32_t *seq_order; /* NULL, or a DEVICE permutation of [0, num_seqs): the order in which
                                 sequences are scheduled (see pa_prefix_order); results do not
                                 depend on it.  Entries outside [0, num_seqs) are skipped and
                                 flagged (PA_DEVERR_CONTEXT); a sequence it does not list gets
                                 no defined output */
} pa_decode_opts;

/* Workspace bytes pa_decode_ext needs (0 = none), (size_t)-1 for invalid
 * dims or options. */
size_t pa_decode_ext_workspace_size(const pa_dims *dims, const pa_decode_opts *opts, int32_t max_context_len,
                                    int32_t partition_tokens);

/*
 * Multi-token / sliding-window decode over a 16-bit or FP8 E4M3 cache
 * (dims->kv_dtype).  q and out are [num_seqs, q_len, num_heads, head_dim] in
 * dims->dtype.  The q_len query tokens of sequence s are its last q_len
 * tokens, already written to the cache: query i sits at position
 * p = context_lens[s] - q_len + i and attends to positions j with
 *     lo <= j <= p,   lo = window > 0 ? max(0, p - window + 1) : 0,
 *     out[s, i, h, :] = sum_j softmax_j(scale * q[s, i, h, :] . K_s[j] * k_scale)
 *                       * V_s[j] * v_scale
 * (a query with p < 0 gets a zero row).  Only the blocks holding attended
 * positions are read: table entries of blocks before a sequence's window
 * may hold anything.  With q_len = 1, window = 0 and unit scales the result
 * is pa_decode's.  max_context_len bounds context_lens as in pa_decode; the
 * workspace is pa_decode_ext_workspace_size bytes.  Errors: those of
 * pa_decode, plus PA_ERR_NULL for opts, PA_ERR_SHAPE for q_len < 1,
 * window < 0 or a scale that is not finite and positive, PA_ERR_UNSUPPORTED
 * for group * q_len > 16.
 */
pa_status pa_decode_ext(void *out, const void *q, const void *k_cache, const void *v_cache,
                        const int32_t *block_tables, const int32_t *context_lens, float scale,
                        int32_t num_kv_heads, const pa_dims *dims, const pa_decode_opts *opts,
                        int32_t max_context_len, int32_t partition_tokens, void *workspace,
                        size_t workspace_bytes, void *stream);

/*
 * Prefix caching, host side ("vLLM PagedAttention 大模型推理架构深度实战"
 * section 7.3: requests with an identical prefix are recognised and share
 * KV-cache blocks; section 2.3: a block's reference count is the number of
 * sequences mapping it).  A table from the content of a full 16-token block
 * (its token ids, chained to the block holding the previous 16 tokens) to the
 * physical block holding its K/V.  Host memory and host pointers only; not
 * thread-safe (one owner, like the block manager that calls it).
 *
 * create:  a cache for block ids [0, num_blocks); NULL on error.
 * match:   the longest chain of cached full blocks equal to the first tokens
 *          of `tokens`; writes their ids to blocks_out (at most max_blocks),
 *          takes one reference on each and returns how many (>= 0), or a
 *          negative pa_status.
 * insert:  registers the full blocks of a sequence (block i holds tokens
 *          [16 i, 16 i + 16)); a block whose prefix is cached already is
 *          left out (the cached one stays canonical); new entries hold one
 *          reference (the inserting sequence's).
 * release: drops one reference on each cached block given (others are
 *          ignored); returns how many were cached.  A block with no
 *          reference stays cached and becomes evictable.
 * evict:   removes up to max_blocks evictable blocks, least recently
 *          released first, writes their ids (free for reuse) and returns how
 *          many.  Their descendants can no longer be matched.
 * stats:   number of cached and evictable blocks, hits and lookups so far.
 */
typedef struct pa_prefix_cache pa_prefix_cache;
pa_prefix_cache *pa_prefix_cache_create(int64_t num_blocks);
void pa_prefix_cache_destroy(pa_prefix_cache *cache);
int32_t pa_prefix_cache_match(pa_prefix_cache *cache, const int32_t *tokens, int32_t num_tokens,
                              int32_t *blocks_out, int32_t max_blocks);
pa_status pa_prefix_cache_insert(pa_prefix_cache *cache, const int32_t *tokens, int32_t num_tokens,
                                 const int32_t *blocks, int32_t num_blocks);
int32_t pa_prefix_cache_release(pa_prefix_cache *cache, const int32_t *blocks, int32_t num_blocks);
int32_t pa_prefix_cache_evict(pa_prefix_cache *cache, int32_t max_blocks, int32_t *blocks_out);
pa_status pa_prefix_cache_stats(const pa_prefix_cache *cache, int64_t *cached, int64_t *evictable,
                                int64_t *hits, int64_t *lookups);

/*
 * Shared-prefix-aware schedule (host): order[i] = the i-th sequence decode
 * should visit, grouping sequences that share their first block (and so
 * their cached prefix) so that their CTAs run together and the shared
 * blocks are read from HBM once and then served from L2.  Sort key: (first
 * block id, sequence index); empty contexts last.  block_tables [num_seqs,
 * max_blocks_per_seq] and context_lens are HOST arrays; order is a host
 * array of num_seqs.  Pass it (copied to the device) as
 * pa_decode_opts.seq_order.
 */
pa_status pa_prefix_order(const int32_t *block_tables, const int32_t *context_lens, int32_t num_seqs,
                          int32_t max_blocks_per_seq, int32_t *order);

/*
 * Cache write (ybb.press section 六, "write into the KV cache block").
 * For every token t < num_tokens with slot = slot_mapping[t] >= 0 and every
 * KV head h:
 *     k_cache[slot / 16, h, slot % 16, :] = key[t, h, :]   (same for value)
 * Negative slots are skipped (padding tokens).  Slots must be distinct: two
 * tokens writing one slot race.  Bit-exact copy; one kernel on `stream`.
 */
pa_status pa_reshape_and_cache(const void *key, const void *value, void *k_cache, void *v_cache,
                               const int64_t *slot_mapping, int32_t num_tokens,
                               const pa_dims *dims, void *stream);

/*
 * Copy-on-write block duplication (ybb.press section 2.3).  For every layer
 * l < num_layers and pair i < num_pairs, (src, dst) = block_mapping[i]:
 *     k_caches[l][dst] = k_caches[l][src]   (all num_kv_heads * 16 * head_dim
 *     v_caches[l][dst] = v_caches[l][src]    elements of the block)
 * k_caches / v_caches are HOST arrays of num_layers device pointers, each
 * cache shaped by dims.  block_mapping is a DEVICE array.  Pairs run
 * concurrently: destinations must be distinct and no destination may also
 * be a source.  Bit-exact; one kernel per 64 layers on `stream`.
 */
pa_status pa_copy_blocks(void *const *k_caches, void *const *v_caches, int32_t num_layers,
                         const int64_t *block_mapping, int32_t num_pairs, const pa_dims *dims,
                         void *stream);

/*
 * Swap blocks between two pools ("vLLM PagedAttention 大模型推理架构深度实战"
 * section 3.2: under memory pressure a low-priority sequence's KV cache is
 * swapped out to CPU memory and resumed later; section 九 item 5: swapped-out
 * KV kept in fast host memory).  For every pair i < num_pairs,
 * (src, dst) = block_mapping[i]:
 *     dst_k[dst] = src_k[src],   dst_v[dst] = src_v[src]
 * (all num_kv_heads * 16 * head_dim elements of a block; dims gives the block
 * geometry and dims->kv_dtype the element size, dims->num_blocks is not used).  The source pools hold
 * src_num_blocks blocks, the destination pools dst_num_blocks.  Each pool may
 * be device memory or page-locked host memory the device can address with
 * the same pointer (cudaHostAlloc / cudaHostRegister under unified
 * addressing): device -> host swaps out, host -> device swaps in.
 * block_mapping [num_pairs, 2] int64 is device or page-locked host memory.
 * Every pointer is checked on the host (cudaPointerGetAttributes): pageable
 * host memory is refused with PA_ERR_MEMORY before anything is enqueued.
 * One kernel moves every pair; destinations must be distinct.  Bit-exact.
 * Out-of-range ids are skipped and flagged (PA_DEVERR_COPY_PAIR).
 */
pa_status pa_swap_blocks(const void *src_k, const void *src_v, int64_t src_num_blocks, void *dst_k,
                         void *dst_v, int64_t dst_num_blocks, const int64_t *block_mapping,
                         int32_t num_pairs, const pa_dims *dims, void *stream);

/*
 * Diagnostic of the failure path: enqueues on `stream` one kernel whose
 * single pipeline wait can never complete (an mbarrier nothing arrives on),
 * bounded to about `milliseconds` (1..2000) of SM clock at the device's
 * maximum clock rate.  The wait gives up, sets PA_DEVERR_TIMEOUT in the
 * device error word and the kernel returns: the context stays usable.  Every
 * pipeline wait of the decode kernels is bounded the same way (about 2 s).
 * Read the word with pa_device_error.
 */
pa_status pa_check_wait_timeout(int32_t milliseconds, void *stream);

/* Thread-local description of the last non-OK status returned on this
 * thread ("" if none).  Owned by the library; valid until the next call. */
const char *pa_last_error(void);

/*
 * Synchronises `stream`, then returns the device error word of the current
 * device (a PA_DEVERR_* bit mask, 0 = clean) through *word and clears it.
 * Returns PA_ERR_CUDA if the synchronisation or the read fails.
 */
pa_status pa_device_error(void *stream, uint32_t *word);

/* Library version: major * 10000 + minor * 100 + patch. */
int32_t pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */
