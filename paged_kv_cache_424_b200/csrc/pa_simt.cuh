// pa_simt.cuh -- the CUDA-core work of decode attention on one KV block,
// used by the decode kernels.
//
// One warp consumes one 16-token block of one KV head that sits in shared
// memory as two contiguous chunks (K then V, each 16 rows x D elements), and
// folds it into the online-softmax state of the G query heads that share the
// KV head ("vLLM PagedAttention 大模型推理架构深度实战" section 5.1: blocks of
// exact attention combined by online softmax):
//   x_t   = q . k_t                    (q pre-scaled by scale * log2 e)
//   m'    = max(m, max_t x_t)   when some x_t > m + kLazyMax, else m' = m
//   l'    = l * 2^(m - m') + sum_t 2^(x_t - m')
//   acc'  = acc * 2^(m - m') + sum_t 2^(x_t - m') v_t
// The final output acc / l does not depend on which m was used; keeping m
// within kLazyMax of the running maximum only bounds the weights.
// Only the first `nvalid` rows of the block are part of the context: the
// others are masked to weight 0 and their V rows are never read.
#pragma once

#include <type_traits>

#include "pa_common.cuh"
#include "pa_decode.h"

namespace pa {

constexpr int kBlock = 16;  // tokens per KV block

// Context length of sequence s, clamped to [0, lmax]; out-of-range values
// are flagged (once per sequence when `report`).
__device__ __forceinline__ int checked_len(const DecodeParams &p, int s, int lmax, bool report) {
    int L = p.context_lens[s];
    if (L < 0 || L > lmax) {
        if (report) flag_error(PA_DEVERR_CONTEXT);
        L = L < 0 ? 0 : lmax;
    }
    return L;
}

// Physical block id read from a table entry, replaced by 0 and flagged when
// outside the pool (it is never dereferenced as given).
__device__ __forceinline__ int64_t checked_block(const DecodeParams &p, int32_t b) {
    if (b < 0 || (int64_t)b >= p.num_blocks) {
        flag_error(PA_DEVERR_BLOCK_ID);
        return 0;
    }
    return b;
}

// The sequence CTA row z works on: z itself, or seq_order[z]; -1 (flagged)
// for an entry outside the batch.
__device__ __forceinline__ int scheduled_seq(const DecodeParams &p, int z, bool report) {
    if (!p.seq_order) return z;
    const int s = p.seq_order[z];
    if (s < 0 || s >= p.num_seqs) {
        if (report) flag_error(PA_DEVERR_CONTEXT);
        return -1;
    }
    return s;
}

// First table entry any query of a sequence of L tokens reads: 0, or with a
// sliding window the block holding the earliest attended position (that of
// query token 0, L - q_len - window + 1).
__device__ __forceinline__ int first_block(const DecodeParams &p, int L) {
    if (p.window <= 0) return 0;
    const int lo = L - p.q_len - p.window + 1;
    return lo > 0 ? lo / kBlock : 0;
}

// How sequence s is split: its checked length, its first block, its blocks
// and its partitions (table entries [bfirst + i * part_blocks, ...) for
// partition i).  Every decode kernel and the merge use this one rule.
struct SeqSplit {
    int L, bfirst, nblk, nparts;
};
__device__ __forceinline__ SeqSplit seq_split(const DecodeParams &p, int s, bool report) {
    SeqSplit r;
    const bool masked = p.q_len != 1 || p.window != 0;
    const int lmax_table = p.max_blocks_per_seq * kBlock;
    r.L = checked_len(p, s, masked ? lmax_table : min(lmax_table, p.max_parts * p.part_blocks * kBlock), report);
    r.nblk = (r.L + kBlock - 1) / kBlock;
    r.bfirst = first_block(p, r.L);
    r.nparts = r.nblk == 0 ? 1 : (r.nblk - r.bfirst + p.part_blocks - 1) / p.part_blocks;
    if (r.nparts > p.max_parts) {  // longer than the plan's max_context_len: flagged, cut
        if (report) flag_error(PA_DEVERR_CONTEXT);
        r.nparts = p.max_parts;
    }
    return r;
}

// Flat index of query row r of KV head kvh of sequence s in q / out ([S,
// q_len, H] rows): query token r / group, head kvh * group + r % group.
__device__ __forceinline__ int64_t query_row(const DecodeParams &p, int s, int kvh, int r) {
    return ((int64_t)s * p.q_len + r / p.group) * p.num_heads + kvh * p.group + r % p.group;
}

// Attended positions [lo, hi] of query row r of a sequence of L tokens
// (hi < 0: none; rows past group * q_len are padding and attend nothing).
__device__ __forceinline__ void row_range(const DecodeParams &p, int L, int r, int *lo, int *hi) {
    const int h = r < p.group * p.q_len ? L - p.q_len + r / p.group : -1;
    *hi = h;
    *lo = p.window > 0 && h - p.window + 1 > 0 ? h - p.window + 1 : 0;
}

// Query rows of a KV-head group in shared memory: fp32, pre-scaled into the
// log2 domain, laid out [h][half][chunk][12] (8 used + 4 pad floats per
// 8-element chunk) so the rotated chunk reads of simt_block are free of
// bank conflicts.
template <int D>
struct SimtQ {
    static constexpr int kNC = D / 16;         // 8-element chunks per half row
    static constexpr int kHalf = kNC * 12;      // floats per padded half row
    static constexpr int floats(int G) { return G * 2 * kHalf; }
};

template <typename T, int D, int G>
__device__ __forceinline__ void load_q_scaled(float *q_s, const T *q_rows, float scale_log2, int tid, int nthreads) {
    for (int i = tid; i < G * D / 2; i += nthreads) {
        const int h = i / (D / 2), e2 = (i % (D / 2)) * 2;
        const uint32_t bits = *reinterpret_cast<const uint32_t *>(q_rows + h * D + e2);
        const float2 f = Elem<T>::to_float2(bits);
        const int half = e2 / (D / 2), e = e2 % (D / 2);
        float *dst = q_s + (h * 2 + half) * SimtQ<D>::kHalf + (e / 8) * 12 + (e % 8);
        dst[0] = f.x * scale_log2;
        dst[1] = f.y * scale_log2;
    }
}

// The same for rows spread over several query tokens: row r is
// q[query_row(p, s, kvh, r)]; padding rows (r >= group * q_len) are zero.
template <typename T, int D, int G>
__device__ __forceinline__ void load_q_rows_scaled(float *q_s, const DecodeParams &p, int s, int kvh, int tid,
                                                   int nthreads) {
    const T *q = reinterpret_cast<const T *>(p.q);
    const int rows = p.group * p.q_len;
    for (int i = tid; i < G * D / 2; i += nthreads) {
        const int h = i / (D / 2), e2 = (i % (D / 2)) * 2;
        float2 f = make_float2(0.f, 0.f);
        if (h < rows) f = Elem<T>::to_float2(*reinterpret_cast<const uint32_t *>(q + query_row(p, s, kvh, h) * D + e2));
        const int half = e2 / (D / 2), e = e2 % (D / 2);
        float *dst = q_s + (h * 2 + half) * SimtQ<D>::kHalf + (e / 8) * 12 + (e % 8);
        dst[0] = f.x * p.scale_log2;
        dst[1] = f.y * p.scale_log2;
    }
}

// Per-warp online-softmax state.  m is kept lazily: it is raised only when a
// logit exceeds it by more than kLazyMax (log2 units), so weights 2^(x - m)
// stay below 2^kLazyMax and most blocks need no max reduction or rescale.
// l is kept as per-lane partial sums (lanes with half == 0 add their token's
// weight) and reduced once by finish().
constexpr float kLazyMax = 8.f;

template <int D, int G>
struct SimtState {
    static constexpr int kPV = D / 32;  // output dims per lane
    float m[G], l[G], acc[G][kPV];
    __device__ __forceinline__ void init() {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            m[h] = -INFINITY;
            l[h] = 0.f;
#pragma unroll
            for (int e = 0; e < kPV; ++e) acc[h][e] = 0.f;
        }
    }
    // Sum the per-lane partial l over the warp (call once, after the last block).
    __device__ __forceinline__ void finish() {
#pragma unroll
        for (int h = 0; h < G; ++h) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) l[h] += __shfl_xor_sync(0xffffffffu, l[h], o);
        }
    }
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// One warp folds one block into `st`.  ks / vs: the K and V chunks in shared
// memory, elements of KT (T itself, or E4M3 codes whose scale the caller
// folds into q and the output); pw: this warp's G x 16 float scratch for the
// softmax weights.
// With kMasked, row h sees only positions lo[h] .. hi[h]; `base` is the
// block's first position.
template <typename T, typename KT, int D, int G, bool kMasked = false>
__device__ __forceinline__ void simt_block(SimtState<D, G> &st, const unsigned char *ks, const unsigned char *vs,
                                           int nvalid, const float *q_s, float *pw, int lane, int base = 0,
                                           const int *lo = nullptr, const int *hi = nullptr) {
    using E = Elem<T>;
    constexpr bool kFp8 = std::is_same<KT, E4M3>::value;
    constexpr int kEsz = kFp8 ? 1 : 2;   // bytes per cache element
    constexpr int kNC = SimtQ<D>::kNC;
    constexpr int kPV = SimtState<D, G>::kPV;
    constexpr int NA = G >= 4 ? 1 : 4 / G;  // independent partial sums per head
    const int t = lane >> 1, half = lane & 1;

    // logits: the lane pair (2t, 2t+1) splits token t's D dims in halves;
    // lanes start at rotated chunks so a warp's 16-byte reads hit 8 distinct
    // bank groups.
    float x[G][NA];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int a = 0; a < NA; ++a) x[h][a] = 0.f;
    const unsigned char *krow = ks + t * D * kEsz + half * (D / 2) * kEsz;
    auto fma8 = [&](const float *k, int qchunk) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float *qc = q_s + (h * 2 + half) * SimtQ<D>::kHalf + qchunk * 12;
            const float4 qa = *reinterpret_cast<const float4 *>(qc);
            const float4 qb = *reinterpret_cast<const float4 *>(qc + 4);
            float *a = x[h];
            a[0 % NA] = fmaf(k[0], qa.x, a[0 % NA]);
            a[1 % NA] = fmaf(k[1], qa.y, a[1 % NA]);
            a[2 % NA] = fmaf(k[2], qa.z, a[2 % NA]);
            a[3 % NA] = fmaf(k[3], qa.w, a[3 % NA]);
            a[0 % NA] = fmaf(k[4], qb.x, a[0 % NA]);
            a[1 % NA] = fmaf(k[5], qb.y, a[1 % NA]);
            a[2 % NA] = fmaf(k[6], qb.z, a[2 % NA]);
            a[3 % NA] = fmaf(k[7], qb.w, a[3 % NA]);
        }
    };
    if constexpr (!kFp8) {
        // 16-byte reads of 8 elements; rotated start per lane
#pragma unroll
        for (int i = 0; i < kNC; ++i) {
            const int c = (i + lane) & (kNC - 1);
            const uint4 raw = *reinterpret_cast<const uint4 *>(krow + c * 16);
            float k[8];
            const float2 k0 = E::to_float2(raw.x), k1 = E::to_float2(raw.y);
            const float2 k2 = E::to_float2(raw.z), k3 = E::to_float2(raw.w);
            k[0] = k0.x; k[1] = k0.y; k[2] = k1.x; k[3] = k1.y;
            k[4] = k2.x; k[5] = k2.y; k[6] = k3.x; k[7] = k3.y;
            fma8(k, c);
        }
    } else {
        // 16-byte reads of 16 E4M3 codes (two 8-element q chunks each)
        constexpr int kNC16 = D / 32;
#pragma unroll
        for (int i = 0; i < kNC16; ++i) {
            const int c = (i + lane) & (kNC16 - 1);
            const uint4 raw = *reinterpret_cast<const uint4 *>(krow + c * 16);
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
            float k[16];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint16_t l16, h16;
                split_b32(w[j], l16, h16);
                const float2 lo = e4m3x2_to_float2(l16);
                const float2 hi = e4m3x2_to_float2(h16);
                k[4 * j] = lo.x; k[4 * j + 1] = lo.y; k[4 * j + 2] = hi.x; k[4 * j + 3] = hi.y;
            }
            fma8(k, 2 * c);
            fma8(k + 8, 2 * c + 1);
        }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float v = x[h][0];
#pragma unroll
        for (int a = 1; a < NA; ++a) v += x[h][a];
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        bool live = t < nvalid;
        if constexpr (kMasked) live = live && base + t >= lo[h] && base + t <= hi[h];
        v = live ? v : -INFINITY;
        if (__any_sync(0xffffffffu, v > st.m[h] + kLazyMax)) {
            // rare: raise the running max to this block's max and rescale
            float bm = v;
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
            const float mn = fmaxf(st.m[h], bm);
            const float alpha = ex2(st.m[h] - mn);  // 0 on the first block (m = -inf)
            st.l[h] *= alpha;
#pragma unroll
            for (int e = 0; e < kPV; ++e) st.acc[h][e] *= alpha;
            st.m[h] = mn;
        }
        // masked rows may still have m = -inf: their weight is 0, not 2^(-inf + inf)
        const float pr = (kMasked && v == -INFINITY) ? 0.f : ex2(v - st.m[h]);
        if (half == 0) {
            st.l[h] += pr;
            pw[h * kBlock + t] = pr;
        }
    }
    __syncwarp();

    // P V: lane owns output dims [lane * kPV, lane * kPV + kPV)
    auto v_row = [&](int tok, float *vf) {
        if constexpr (kFp8) {
            if constexpr (kPV == 4) {
                const uint32_t raw = *reinterpret_cast<const uint32_t *>(vs + tok * D + lane * 4);
                uint16_t l16, h16;
                split_b32(raw, l16, h16);
                const float2 a = e4m3x2_to_float2(l16);
                const float2 b = e4m3x2_to_float2(h16);
                vf[0] = a.x;
                vf[1] = a.y;
                vf[2] = b.x;
                vf[3] = b.y;
            } else {
                const float2 a = e4m3x2_to_float2(*reinterpret_cast<const uint16_t *>(vs + tok * D + lane * 2));
                vf[0] = a.x;
                vf[1] = a.y;
            }
        } else if constexpr (kPV == 4) {
            const uint2 raw = *reinterpret_cast<const uint2 *>(vs + tok * D * 2 + lane * 8);
            const float2 a = E::to_float2(raw.x), b = E::to_float2(raw.y);
            vf[0] = a.x;
            vf[1] = a.y;
            vf[2] = b.x;
            vf[3] = b.y;
        } else {
            const uint32_t raw = *reinterpret_cast<const uint32_t *>(vs + tok * D * 2 + lane * 4);
            const float2 a = E::to_float2(raw);
            vf[0] = a.x;
            vf[1] = a.y;
        }
    };
    if (nvalid == kBlock) {
        // full block: straight-line code so the 16 row loads issue back to back
        float vf[kBlock][kPV];
#pragma unroll
        for (int tok = 0; tok < kBlock; ++tok) v_row(tok, vf[tok]);
#pragma unroll
        for (int h = 0; h < G; ++h) {
#pragma unroll
            for (int tq = 0; tq < kBlock / 4; ++tq) {
                const float4 pq = *reinterpret_cast<const float4 *>(pw + h * kBlock + tq * 4);
                const float pv[4] = {pq.x, pq.y, pq.z, pq.w};
#pragma unroll
                for (int tt = 0; tt < 4; ++tt)
#pragma unroll
                    for (int e = 0; e < kPV; ++e) st.acc[h][e] = fmaf(pv[tt], vf[tq * 4 + tt][e], st.acc[h][e]);
            }
        }
    } else {
        // the sequence's last block: only its first nvalid rows exist
        for (int tok = 0; tok < nvalid; ++tok) {
            float vf[kPV];
            v_row(tok, vf);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float pv = pw[h * kBlock + tok];
#pragma unroll
                for (int e = 0; e < kPV; ++e) st.acc[h][e] = fmaf(pv, vf[e], st.acc[h][e]);
            }
        }
    }
    __syncwarp();
}

// Cross-warp combination of NW warp states stored as red_m/red_l [NW][G] and
// red_acc [NW][G][D]: for element (h, d) returns o = sum_w 2^(m_w - M) acc_w /
// sum_w 2^(m_w - M) l_w and lse = M + log2(sum_w 2^(m_w - M) l_w).  Warps
// that saw no block have m = -inf and l = acc = 0 and drop out; a row that
// no warp saw (possible only with masks) gives o = 0, lse = -inf.
template <int D, int G, int NW>
__device__ __forceinline__ float combine_warps(const float *red_m, const float *red_l, const float *red_acc, int h,
                                               int d, float *lse) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, red_m[w * G + h]);
    if (M == -INFINITY) {  // a masked row with no position in this partition
        *lse = -INFINITY;
        return 0.f;
    }
    float lsum = 0.f, o = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        const float f = exp2f(red_m[w * G + h] - M);
        lsum = fmaf(red_l[w * G + h], f, lsum);
        o = fmaf(red_acc[(w * G + h) * D + d], f, o);
    }
    *lse = M + log2f(lsum);
    return o / lsum;
}

}  // namespace pa
