/*
 * pa_oracle.c -- plain, slow, double-precision CPU oracle for paged decode
 * attention and its two companion cache operations.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the package smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA library; the two meet only at the documented memory layouts.
 *
 * What it follows (sources are the web pages this library is built from):
 *  - "vLLM PagedAttention 大模型推理架构深度实战" (ybb.press), section 2.2
 *    "PagedAttention核心机制": the KV cache is cut into fixed blocks of 16
 *    tokens; each sequence owns a block table that maps its logical block
 *    index to a physical block, like an OS page table.
 *  - "vLLM：重塑大模型推理性能的关键引擎" (unionyoga.cn), section
 *    "vLLM 如何破局？从PagedAttention说起", kernel sketch: a sequence needs
 *    ceil(context_len / BLOCK_SIZE) blocks; logical block i of sequence s is
 *    block_table[s * MAX_BLOCKS + i].
 *  - The same ybb.press page, section 2.1 and section 5.1: decode attention
 *    of a new token against all cached keys/values is exact attention,
 *    softmax(q K^T * scale) V.  No approximation is involved, so this oracle
 *    is that definition written out (two-pass, max-subtracted softmax, which
 *    is the same function), not the online/blocked algorithm the GPU runs.
 *  - ybb.press section 2.3 "写时复制与并行采样": a shared block is copied
 *    before a sharer modifies it; copy_blocks is a plain byte copy.
 *  - ybb.press section 六 "架构总览" (decode loop): each iteration writes the
 *    new token's K/V into its KV-cache block; reshape_and_cache is the plain
 *    indexed assignment.
 *  - ybb.press section 3.2 (preemption: a sequence's KV cache is swapped out
 *    to CPU memory and resumed later) and section 九 item 5 (swapped-out KV
 *    kept in fast host memory): swap_blocks is a block copy between two
 *    pools.
 *
 * Layouts (row-major, contiguous; element = 16-bit fp16 or bf16 bit pattern):
 *   q, out        [num_seqs, num_heads, head_dim]   (out is double here)
 *   k/v cache     [num_blocks, num_kv_heads, block_size, head_dim]
 *   block_tables  [num_seqs, max_blocks_per_seq] int32
 *   context_lens  [num_seqs] int32
 *   key/value     [num_tokens, num_kv_heads, head_dim]
 *   slot_mapping  [num_tokens] int64, slot = block * block_size + offset,
 *                 negative = skip
 *   block_mapping [num_pairs, 2] int64 (src, dst)
 *
 * FP8 KV cache (a later variant of the same path; the pages name FP8 only
 * for weights, ybb.press section 5.2, and KV-cache compression as a goal,
 * section 九 item 3): caches of OCP FP8 E4M3 codes (bias 7, 3 mantissa
 * bits, no infinities, S.1111.111 = NaN, largest finite 448) with one fp32
 * scale per tensor: element = decode(code) * scale.  Quantisation of a
 * 16-bit value x: y = float(x) / scale in IEEE fp32 (one correctly rounded
 * division), then the E4M3 value nearest to y, ties to the even code,
 * magnitudes beyond 448 clamped to 448 ("saturate to finite"), NaN -> NaN.
 *
 * Readings where the pages are silent: query head h reads KV head
 * h / (num_heads / num_kv_heads) (contiguous GQA groups); a context length of
 * zero yields an all-zero output row.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_ARG (-1)
#define ORC_ERR_RANGE (-2)
#define ORC_ERR_NOMEM (-3)

#define ORC_F16 0
#define ORC_BF16 1

/* IEEE 754 binary16 -> double, exactly: sign, 5-bit exponent (bias 15),
 * 10-bit fraction; exponent 0 is subnormal (fraction * 2^-24). */
static double widen_f16(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m + 1024), e - 25);
    return sign ? -v : v;
}

/* bfloat16 is the top half of an IEEE binary32: put it back and widen. */
static double widen_bf16(uint16_t h) {
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static double widen(uint16_t h, int32_t dtype) {
    return dtype == ORC_BF16 ? widen_bf16(h) : widen_f16(h);
}

/* OCP FP8 E4M3 code -> double: sign, 4-bit exponent (bias 7), 3-bit
 * fraction; exponent 0 is subnormal (fraction * 2^-9); code S.1111.111 is
 * NaN (there are no infinities). */
static double widen_e4m3(uint8_t c) {
    int sign = (c >> 7) & 1;
    int e = (c >> 3) & 0xf;
    int m = c & 7;
    double v;
    if (e == 15 && m == 7)
        v = NAN;
    else if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp((double)(m + 8), e - 10);
    return sign ? -v : v;
}

/* Magnitudes of the positive finite E4M3 codes 0x01 .. 0x7e, in code order
 * (which is ascending order of value), widened once per call so that the
 * nearest-code search below reads a table instead of re-widening. */
typedef struct {
    double v[0x7f];
} e4m3_table;

static void e4m3_table_fill(e4m3_table *t) {
    for (int c = 0; c < 0x7f; ++c) t->v[c] = widen_e4m3((uint8_t)c);
}

/* Nearest E4M3 code to y (ties to the even code), clamped to +-448: a
 * search over every positive finite code for |y|, then y's sign (so -0.0
 * and negatives that round to zero give -0, code 0x80). */
static uint8_t quantize_e4m3(float y, const e4m3_table *t) {
    if (y != y) return 0x7f;
    double a = fabs((double)y);
    uint8_t best = 0;
    double best_err = a;  /* code 0 = +0 */
    for (uint8_t c = 1; c < 0x7f; ++c) {  /* every positive finite code, ascending */
        double err = fabs(t->v[c] - a);
        if (err < best_err || (err == best_err && (c & 1) == 0)) {
            best = c;
            best_err = err;
        }
    }
    if (a > 448.0) best = 0x7e;  /* saturate to finite */
    return (uint8_t)(best | (signbit(y) ? 0x80 : 0));  /* the sign is kept, -0 included */
}

void oracle_quantize_e4m3_n(uint8_t *out, const float *y, int64_t n) {
    e4m3_table t;
    e4m3_table_fill(&t);
    for (int64_t i = 0; i < n; ++i) out[i] = quantize_e4m3(y[i], &t);
}
void oracle_widen_e4m3_n(double *out, const uint8_t *c, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = widen_e4m3(c[i]);
}

int oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Decode attention for every (sequence, query head).
 *
 * For sequence s with n = context_lens[s] tokens and query head h
 * (KV head kvh = h / group):
 *   K_s[j] = k_cache[block_tables[s, j / block_size], kvh, j % block_size, :]
 *   x_j    = scale * sum_d q[s, h, d] * K_s[j, d]                (j < n)
 *   out[s, h, :] = sum_j softmax(x)_j * V_s[j, :]
 * Only slots j < n are read: the tail of the last block and the table
 * entries past ceil(n / block_size) are never touched.
 */
int oracle_paged_decode(double *out, const uint16_t *q, const uint16_t *k_cache,
                        const uint16_t *v_cache, const int32_t *block_tables,
                        const int32_t *context_lens, double scale, int32_t num_seqs,
                        int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                        int32_t block_size, int32_t max_blocks_per_seq,
                        int64_t num_blocks, int32_t dtype) {
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return ORC_ERR_ARG;
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || max_blocks_per_seq < 0 || num_blocks <= 0)
        return ORC_ERR_ARG;
    if (num_heads % num_kv_heads != 0) return ORC_ERR_ARG;
    if (dtype != ORC_F16 && dtype != ORC_BF16) return ORC_ERR_ARG;

    /* Every referenced block id must lie in the pool. */
    for (int32_t s = 0; s < num_seqs; ++s) {
        int32_t n = context_lens[s];
        if (n < 0 || (int64_t)n > (int64_t)max_blocks_per_seq * block_size) return ORC_ERR_RANGE;
        int32_t nblk = (n + block_size - 1) / block_size;
        for (int32_t i = 0; i < nblk; ++i) {
            int32_t b = block_tables[(int64_t)s * max_blocks_per_seq + i];
            if (b < 0 || (int64_t)b >= num_blocks) return ORC_ERR_RANGE;
        }
    }

    const int32_t group = num_heads / num_kv_heads;
    const int64_t pairs = (int64_t)num_seqs * num_heads;
    int status = ORC_OK;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t p = 0; p < pairs; ++p) {
        const int32_t s = (int32_t)(p / num_heads);
        const int32_t h = (int32_t)(p % num_heads);
        const int32_t kvh = h / group;
        const int32_t n = context_lens[s];
        double *o = out + p * head_dim;
        for (int32_t d = 0; d < head_dim; ++d) o[d] = 0.0;
        if (n == 0) continue;

        double *x = (double *)malloc(sizeof(double) * (size_t)n);
        double *qd = (double *)malloc(sizeof(double) * (size_t)head_dim);
        if (!x || !qd) {
            free(x);
            free(qd);
#pragma omp atomic write
            status = ORC_ERR_NOMEM;
            continue;
        }
        for (int32_t d = 0; d < head_dim; ++d) qd[d] = widen(q[p * head_dim + d], dtype);

        /* Pass 1: logits through the block table. */
        for (int32_t j = 0; j < n; ++j) {
            int64_t blk = block_tables[(int64_t)s * max_blocks_per_seq + j / block_size];
            int64_t row = ((blk * num_kv_heads + kvh) * block_size + j % block_size) * head_dim;
            double dot = 0.0;
            for (int32_t d = 0; d < head_dim; ++d) dot += qd[d] * widen(k_cache[row + d], dtype);
            x[j] = scale * dot;
        }
        /* Softmax: subtract the max (the result is unchanged), normalise. */
        double m = x[0];
        for (int32_t j = 1; j < n; ++j)
            if (x[j] > m) m = x[j];
        double z = 0.0;
        for (int32_t j = 0; j < n; ++j) {
            x[j] = exp(x[j] - m);
            z += x[j];
        }
        /* Pass 2: probability-weighted sum of the values. */
        for (int32_t j = 0; j < n; ++j) {
            int64_t blk = block_tables[(int64_t)s * max_blocks_per_seq + j / block_size];
            int64_t row = ((blk * num_kv_heads + kvh) * block_size + j % block_size) * head_dim;
            double w = x[j] / z;
            for (int32_t d = 0; d < head_dim; ++d) o[d] += w * widen(v_cache[row + d], dtype);
        }
        free(x);
        free(qd);
    }
    return status;
}

/*
 * Cache write: for every token t with slot = slot_mapping[t] >= 0,
 *   k_cache[slot / block_size, h, slot % block_size, :] = key[t, h, :]
 * and the same for value, for every KV head h.  Tokens are applied in order.
 */
int oracle_reshape_and_cache(uint16_t *k_cache, uint16_t *v_cache, const uint16_t *key,
                             const uint16_t *value, const int64_t *slot_mapping,
                             int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                             int32_t block_size, int64_t num_blocks) {
    if (!k_cache || !v_cache || (num_tokens > 0 && (!key || !value || !slot_mapping)))
        return ORC_ERR_ARG;
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
        return ORC_ERR_ARG;
    for (int32_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot / block_size >= num_blocks) return ORC_ERR_RANGE;
    }
    for (int32_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        int64_t blk = slot / block_size, off = slot % block_size;
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * head_dim;
            int64_t src = ((int64_t)t * num_kv_heads + h) * head_dim;
            for (int32_t d = 0; d < head_dim; ++d) {
                k_cache[dst + d] = key[src + d];
                v_cache[dst + d] = value[src + d];
            }
        }
    }
    return ORC_OK;
}

/*
 * Copy-on-write duplication: for every layer and every pair (src, dst),
 * copy all num_kv_heads * block_size * head_dim elements of block src to
 * block dst, in the K and the V cache.  Pairs are applied in order.
 */
int oracle_copy_blocks(uint16_t *const *k_caches, uint16_t *const *v_caches, int32_t num_layers,
                       const int64_t *block_mapping, int32_t num_pairs, int32_t num_kv_heads,
                       int32_t head_dim, int32_t block_size, int64_t num_blocks) {
    if (num_layers < 0 || num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || num_blocks <= 0)
        return ORC_ERR_ARG;
    if ((num_layers > 0 && (!k_caches || !v_caches)) || (num_pairs > 0 && !block_mapping))
        return ORC_ERR_ARG;
    for (int32_t i = 0; i < num_pairs; ++i) {
        int64_t src = block_mapping[2 * i], dst = block_mapping[2 * i + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) return ORC_ERR_RANGE;
    }
    const int64_t elems = (int64_t)num_kv_heads * block_size * head_dim;
    for (int32_t l = 0; l < num_layers; ++l) {
        if (!k_caches[l] || !v_caches[l]) return ORC_ERR_ARG;
        for (int32_t i = 0; i < num_pairs; ++i) {
            int64_t src = block_mapping[2 * i], dst = block_mapping[2 * i + 1];
            memmove(k_caches[l] + dst * elems, k_caches[l] + src * elems, sizeof(uint16_t) * elems);
            memmove(v_caches[l] + dst * elems, v_caches[l] + src * elems, sizeof(uint16_t) * elems);
        }
    }
    return ORC_OK;
}

/*
 * Swap between two pools: for every pair (src, dst), block dst of the
 * destination K and V pools becomes a copy of block src of the source pools.
 */
int oracle_swap_blocks(uint16_t *dst_k, uint16_t *dst_v, int64_t dst_num_blocks, const uint16_t *src_k,
                       const uint16_t *src_v, int64_t src_num_blocks, const int64_t *block_mapping,
                       int32_t num_pairs, int32_t num_kv_heads, int32_t head_dim, int32_t block_size) {
    if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0) return ORC_ERR_ARG;
    if (num_pairs > 0 && (!dst_k || !dst_v || !src_k || !src_v || !block_mapping)) return ORC_ERR_ARG;
    for (int32_t i = 0; i < num_pairs; ++i) {
        int64_t src = block_mapping[2 * i], dst = block_mapping[2 * i + 1];
        if (src < 0 || src >= src_num_blocks || dst < 0 || dst >= dst_num_blocks) return ORC_ERR_RANGE;
    }
    const int64_t elems = (int64_t)num_kv_heads * block_size * head_dim;
    for (int32_t i = 0; i < num_pairs; ++i) {
        int64_t src = block_mapping[2 * i], dst = block_mapping[2 * i + 1];
        memcpy(dst_k + dst * elems, src_k + src * elems, sizeof(uint16_t) * elems);
        memcpy(dst_v + dst * elems, src_v + src * elems, sizeof(uint16_t) * elems);
    }
    return ORC_OK;
}

/*
 * Decode attention over FP8 E4M3 caches with per-tensor scales: the same
 * definition as oracle_paged_decode, with K_s[j, d] = decode(k_code) * k_scale
 * and V_s[j, d] = decode(v_code) * v_scale; q and out as before (q_dtype).
 */
int oracle_paged_decode_fp8(double *out, const uint16_t *q, const uint8_t *k_cache, const uint8_t *v_cache,
                            const int32_t *block_tables, const int32_t *context_lens, double scale,
                            double k_scale, double v_scale, int32_t num_seqs, int32_t num_heads,
                            int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                            int32_t max_blocks_per_seq, int64_t num_blocks, int32_t q_dtype) {
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return ORC_ERR_ARG;
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        max_blocks_per_seq < 0 || num_blocks <= 0 || num_heads % num_kv_heads != 0)
        return ORC_ERR_ARG;
    if (q_dtype != ORC_F16 && q_dtype != ORC_BF16) return ORC_ERR_ARG;
    for (int32_t s = 0; s < num_seqs; ++s) {
        int32_t n = context_lens[s];
        if (n < 0 || (int64_t)n > (int64_t)max_blocks_per_seq * block_size) return ORC_ERR_RANGE;
        for (int32_t i = 0; i < (n + block_size - 1) / block_size; ++i) {
            int32_t b = block_tables[(int64_t)s * max_blocks_per_seq + i];
            if (b < 0 || (int64_t)b >= num_blocks) return ORC_ERR_RANGE;
        }
    }
    const int32_t group = num_heads / num_kv_heads;
    const int64_t pairs = (int64_t)num_seqs * num_heads;
    int status = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t p = 0; p < pairs; ++p) {
        const int32_t s = (int32_t)(p / num_heads), h = (int32_t)(p % num_heads);
        const int32_t kvh = h / group, n = context_lens[s];
        double *o = out + p * head_dim;
        for (int32_t d = 0; d < head_dim; ++d) o[d] = 0.0;
        if (n == 0) continue;
        double *x = (double *)malloc(sizeof(double) * (size_t)n);
        if (!x) {
#pragma omp atomic write
            status = ORC_ERR_NOMEM;
            continue;
        }
        for (int32_t j = 0; j < n; ++j) {
            int64_t blk = block_tables[(int64_t)s * max_blocks_per_seq + j / block_size];
            int64_t row = ((blk * num_kv_heads + kvh) * block_size + j % block_size) * head_dim;
            double dot = 0.0;
            for (int32_t d = 0; d < head_dim; ++d)
                dot += widen(q[p * head_dim + d], q_dtype) * (widen_e4m3(k_cache[row + d]) * k_scale);
            x[j] = scale * dot;
        }
        double m = x[0];
        for (int32_t j = 1; j < n; ++j)
            if (x[j] > m) m = x[j];
        double z = 0.0;
        for (int32_t j = 0; j < n; ++j) {
            x[j] = exp(x[j] - m);
            z += x[j];
        }
        for (int32_t j = 0; j < n; ++j) {
            int64_t blk = block_tables[(int64_t)s * max_blocks_per_seq + j / block_size];
            int64_t row = ((blk * num_kv_heads + kvh) * block_size + j % block_size) * head_dim;
            double w = x[j] / z;
            for (int32_t d = 0; d < head_dim; ++d) o[d] += w * (widen_e4m3(v_cache[row + d]) * v_scale);
        }
        free(x);
    }
    return status;
}

/*
 * Cache write into FP8 E4M3 caches: for every token t with slot >= 0,
 *   k_cache[slot / block_size, h, slot % block_size, d] =
 *       quantize(float(key[t, h, d]) / k_scale)      (same for value, v_scale)
 */
int oracle_reshape_and_cache_fp8(uint8_t *k_cache, uint8_t *v_cache, const uint16_t *key, const uint16_t *value,
                                 const int64_t *slot_mapping, int32_t num_tokens, int32_t num_kv_heads,
                                 int32_t head_dim, int32_t block_size, int64_t num_blocks, int32_t dtype,
                                 float k_scale, float v_scale) {
    if (!k_cache || !v_cache || (num_tokens > 0 && (!key || !value || !slot_mapping))) return ORC_ERR_ARG;
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
        return ORC_ERR_ARG;
    if (dtype != ORC_F16 && dtype != ORC_BF16) return ORC_ERR_ARG;
    for (int32_t t = 0; t < num_tokens; ++t)
        if (slot_mapping[t] >= 0 && slot_mapping[t] / block_size >= num_blocks) return ORC_ERR_RANGE;
    e4m3_table tab;
    e4m3_table_fill(&tab);
    /* heads write disjoint rows, so they may run in parallel; tokens stay in
     * order within a head */
#pragma omp parallel for schedule(static)
    for (int32_t h = 0; h < num_kv_heads; ++h) {
        for (int32_t t = 0; t < num_tokens; ++t) {
            int64_t slot = slot_mapping[t];
            if (slot < 0) continue;
            int64_t blk = slot / block_size, off = slot % block_size;
            int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * head_dim;
            int64_t src = ((int64_t)t * num_kv_heads + h) * head_dim;
            for (int32_t d = 0; d < head_dim; ++d) {
                k_cache[dst + d] = quantize_e4m3((float)widen(key[src + d], dtype) / k_scale, &tab);
                v_cache[dst + d] = quantize_e4m3((float)widen(value[src + d], dtype) / v_scale, &tab);
            }
        }
    }
    return ORC_OK;
}

/*
 * Multi-token and sliding-window decode (variants of the same path: a
 * sliding-window mask over the same block stream, which "vLLM PagedAttention
 * 大模型推理架构深度实战" section 7.2 recommends for long contexts, and several
 * query tokens per sequence, as the large model's parallel verification of
 * draft tokens in speculative decoding needs, the same page's section 九
 * item 2).  Readings, where the page gives no formula:
 *   - the q_len query tokens of sequence s are its last q_len tokens, whose
 *     K/V are already in the cache: query i sits at position
 *     p_i = context_lens[s] - q_len + i and attends causally to j <= p_i;
 *   - a window of W > 0 tokens keeps the W most recent positions including
 *     the query's own: j >= p_i - W + 1 (W = 0: no window);
 *   - a query with no position to attend to (p_i < 0) gets a zero row.
 * For sequence s, query token i, query head h (KV head kvh = h / group),
 * lo_i = W > 0 ? max(0, p_i - W + 1) : 0:
 *   x_j = scale * sum_d q[s, i, h, d] * K_s[j, d] * k_scale    (lo_i <= j <= p_i)
 *   out[s, i, h, :] = sum_j softmax(x)_j * V_s[j, :] * v_scale
 * K_s / V_s through the block table as in oracle_paged_decode; the cache
 * holds 16-bit elements of `dtype` (kv_fp8 = 0) or E4M3 codes (kv_fp8 = 1).
 * q and out are [num_seqs, q_len, num_heads, head_dim].  Only the blocks
 * holding positions lo_i .. p_i are read (table entries of blocks before the
 * window are never touched).
 */
int oracle_paged_decode_ext(double *out, const uint16_t *q, const void *k_cache, const void *v_cache,
                            const int32_t *block_tables, const int32_t *context_lens, double scale,
                            double k_scale, double v_scale, int32_t num_seqs, int32_t num_heads,
                            int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                            int32_t max_blocks_per_seq, int64_t num_blocks, int32_t dtype, int32_t kv_fp8,
                            int32_t q_len, int32_t window) {
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return ORC_ERR_ARG;
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        max_blocks_per_seq < 0 || num_blocks <= 0 || q_len <= 0 || window < 0)
        return ORC_ERR_ARG;
    if (num_heads % num_kv_heads != 0) return ORC_ERR_ARG;
    if (dtype != ORC_F16 && dtype != ORC_BF16) return ORC_ERR_ARG;
    const uint16_t *k16 = (const uint16_t *)k_cache, *v16 = (const uint16_t *)v_cache;
    const uint8_t *k8 = (const uint8_t *)k_cache, *v8 = (const uint8_t *)v_cache;

    /* Every block id that will be read must lie in the pool. */
    for (int32_t s = 0; s < num_seqs; ++s) {
        int32_t n = context_lens[s];
        if (n < 0 || (int64_t)n > (int64_t)max_blocks_per_seq * block_size) return ORC_ERR_RANGE;
        for (int32_t i = 0; i < q_len; ++i) {
            int32_t hi = n - q_len + i;
            if (hi < 0) continue;
            int32_t lo = window > 0 && hi - window + 1 > 0 ? hi - window + 1 : 0;
            for (int32_t bi = lo / block_size; bi <= hi / block_size; ++bi) {
                int32_t b = block_tables[(int64_t)s * max_blocks_per_seq + bi];
                if (b < 0 || (int64_t)b >= num_blocks) return ORC_ERR_RANGE;
            }
        }
    }

    const int32_t group = num_heads / num_kv_heads;
    const int64_t rows = (int64_t)num_seqs * q_len * num_heads;
    int status = ORC_OK;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        const int32_t s = (int32_t)(r / ((int64_t)q_len * num_heads));
        const int32_t i = (int32_t)(r / num_heads % q_len);
        const int32_t h = (int32_t)(r % num_heads);
        const int32_t kvh = h / group;
        const int32_t hi = context_lens[s] - q_len + i;
        double *o = out + r * head_dim;
        for (int32_t d = 0; d < head_dim; ++d) o[d] = 0.0;
        if (hi < 0) continue;
        const int32_t lo = window > 0 && hi - window + 1 > 0 ? hi - window + 1 : 0;
        const int32_t n = hi - lo + 1;

        double *x = (double *)malloc(sizeof(double) * (size_t)n);
        double *qd = (double *)malloc(sizeof(double) * (size_t)head_dim);
        if (!x || !qd) {
            free(x);
            free(qd);
#pragma omp atomic write
            status = ORC_ERR_NOMEM;
            continue;
        }
        for (int32_t d = 0; d < head_dim; ++d) qd[d] = widen(q[r * head_dim + d], dtype);

        /* logits of positions lo .. hi through the block table */
        for (int32_t j = lo; j <= hi; ++j) {
            int64_t blk = block_tables[(int64_t)s * max_blocks_per_seq + j / block_size];
            int64_t row = ((blk * num_kv_heads + kvh) * block_size + j % block_size) * head_dim;
            double dot = 0.0;
            for (int32_t d = 0; d < head_dim; ++d) {
                double kv = kv_fp8 ? widen_e4m3(k8[row + d]) : widen(k16[row + d], dtype);
                dot += qd[d] * (kv * k_scale);
            }
            x[j - lo] = scale * dot;
        }
        /* softmax (max-subtracted) and the weighted sum of V */
        double m = -INFINITY;
        for (int32_t j = 0; j < n; ++j)
            if (x[j] > m) m = x[j];
        double z = 0.0;
        for (int32_t j = 0; j < n; ++j) {
            x[j] = exp(x[j] - m);
            z += x[j];
        }
        for (int32_t j = lo; j <= hi; ++j) {
            int64_t blk = block_tables[(int64_t)s * max_blocks_per_seq + j / block_size];
            int64_t row = ((blk * num_kv_heads + kvh) * block_size + j % block_size) * head_dim;
            double w = x[j - lo] / z;
            for (int32_t d = 0; d < head_dim; ++d) {
                double vv = kv_fp8 ? widen_e4m3(v8[row + d]) : widen(v16[row + d], dtype);
                o[d] += w * (vv * v_scale);
            }
        }
        free(x);
        free(qd);
    }
    return status;
}
