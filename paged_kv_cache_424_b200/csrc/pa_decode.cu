// pa_decode.cu -- paged decode attention over fixed-size KV partitions
// (CUDA-core path), and its log-sum-exp merge.
//
// Method: "vLLM PagedAttention 大模型推理架构深度实战" section 2.2 (a sequence's
// KV lives in 16-token physical blocks named by its block table) and section
// 5.1 (exact attention, blocks combined by online softmax);
// "vLLM：重塑大模型推理性能的关键引擎", PagedAttention section, kernel sketch
// (ceil(len / 16) blocks, entry i of the table row is logical block i).
//
// Work decomposition:
//   CTA = (KV partition p, KV head kvh, sequence s), 4 warps.  The CTA's
//   partition covers table entries [p * part_blocks, ...).  Warp w takes
//   the partition's blocks w, w + 4, w + 8, ... and streams them through its
//   own NSTAGE-deep ring of shared-memory stages: one lane issues two 1-D
//   bulk copies (the K chunk and the V chunk of (block, kvh), each one
//   contiguous 16 x D x 2-byte run in the head-major pool) that complete on
//   the stage's mbarrier.  Each warp keeps an online-softmax state for the G
//   query heads that share kvh; at the end the 4 warp states are merged in
//   shared memory.  If the sequence needs one partition the CTA writes the
//   output; otherwise it writes (o_p, log2-sum-exp_p) to the workspace and
//   the merge kernel combines partitions:
//     out = sum_p 2^(lse_p - M) o_p / sum_p 2^(lse_p - M),  M = max_p lse_p.
#include <type_traits>

#include "pa_common.cuh"
#include "pa_decode.h"
#include "pa_simt.cuh"

namespace pa {

namespace {

constexpr int kWarps = 4;

// Shared-memory layout of the fixed-partition kernel (bytes):
//   [main]  per-warp stage rings (kWarps x NSTAGE x {K chunk, V chunk}); reused
//           at the end for the cross-warp reduction (kWarps x G x D floats)
//   [q]     padded query rows (SimtQ)
//   [p]     kWarps x G x 16 floats (softmax weights)
//   [m, l]  2 x kWarps x G floats
//   [bars]  kWarps x NSTAGE mbarriers
//   [table] part_blocks int32
struct PartLayout {
    int chunk, main, q_off, p_off, ml_off, bar_off, table_off;
    __host__ __device__ constexpr PartLayout(int D, int G, int nstage, int esz)
        : chunk(kBlock * D * esz),
          main(kWarps * nstage * 2 * kBlock * D * esz > kWarps * G * D * 4 ? kWarps * nstage * 2 * kBlock * D * esz
                                                                          : kWarps * G * D * 4),
          q_off(main), p_off(q_off + G * 2 * (D / 16) * 12 * 4), ml_off(p_off + kWarps * G * kBlock * 4),
          bar_off((ml_off + 2 * kWarps * G * 4 + 7) / 8 * 8), table_off(bar_off + kWarps * nstage * 8) {}
    __host__ __device__ constexpr int bytes(int part_blocks) const { return table_off + part_blocks * 4; }
};

// Stages per warp ring: 2 with small groups (more CTAs per SM, more warps
// to hide the per-block latency chains), 3 otherwise.  FP8 blocks are half
// the bytes, so the same stages let twice the CTAs fit per SM, which keeps
// the bytes in flight and doubles the warps that widen the codes.
__host__ __device__ constexpr int part_stages(int G, int esz) { return (void)esz, G <= 2 ? 2 : 3; }

template <typename T, typename KT, int D, int G, int NSTAGE, bool kMasked>
__global__ void __launch_bounds__(kWarps * 32) decode_part_kernel(const DecodeParams p) {
    constexpr int kEsz = std::is_same<KT, E4M3>::value ? 1 : 2;
    constexpr PartLayout S(D, G, NSTAGE, kEsz);
    using E = Elem<T>;

    extern __shared__ __align__(128) unsigned char smem[];
    float *q_s = reinterpret_cast<float *>(smem + S.q_off);
    float *p_s = reinterpret_cast<float *>(smem + S.p_off);
    float *red_m = reinterpret_cast<float *>(smem + S.ml_off);
    float *red_l = red_m + kWarps * G;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S.bar_off);
    int32_t *tbl = reinterpret_cast<int32_t *>(smem + S.table_off);
    __shared__ int fail_s;

    const int part = blockIdx.x, kvh = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.num_heads;
    const int head0 = kvh * G;  // unmasked launches only (group == G, q_len == 1)
    pdl_launch_dependents();
    pdl_wait();
    const int s = scheduled_seq(p, blockIdx.z, part == 0 && kvh == 0 && tid == 0);
    if (s < 0) return;
    // flat q / out row of row r: plain decode keeps the group's rows contiguous
    auto row_of = [&](int r) -> int64_t {
        if constexpr (kMasked) return query_row(p, s, kvh, r);
        return (int64_t)s * H + head0 + r;
    };
    const int rows = kMasked ? p.group * p.q_len : G;  // real rows (the rest is padding)

    const SeqSplit sp = seq_split(p, s, part == 0 && kvh == 0 && tid == 0);
    const int L = sp.L, nblk = sp.nblk, nparts = sp.nparts;
    if (part >= nparts) return;
    const bool direct = nparts == 1;
    T *out = reinterpret_cast<T *>(p.out);

    if (L == 0) {  // empty context: zero rows
        for (int i = tid; i < rows * D; i += blockDim.x) out[row_of(i / D) * D + i % D] = E::from_float(0.f);
        return;
    }

    int lo[G], hi[G];  // attended positions of each row (masked launches)
#pragma unroll
    for (int r = 0; r < G; ++r) {
        if constexpr (kMasked) {
            row_range(p, L, r, &lo[r], &hi[r]);
        } else {
            lo[r] = 0;
            hi[r] = L - 1;
        }
    }

    const int b0 = sp.bfirst + part * p.part_blocks;
    const int b1 = min(b0 + p.part_blocks, nblk);
    for (int i = tid; i < b1 - b0; i += blockDim.x)
        tbl[i] = (int32_t)checked_block(p, p.block_tables[(int64_t)s * p.max_blocks_per_seq + b0 + i]);
    if constexpr (kMasked)
        load_q_rows_scaled<T, D, G>(q_s, p, s, kvh, tid, blockDim.x);
    else
        load_q_scaled<T, D, G>(q_s, reinterpret_cast<const T *>(p.q) + ((int64_t)s * H + head0) * D, p.scale_log2,
                               tid, blockDim.x);
    if (tid == 0) {
        fail_s = 0;
        for (int i = 0; i < kWarps * NSTAGE; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    __syncthreads();

    // ---- per-warp pipeline -------------------------------------------------
    unsigned char *stages = smem + warp * NSTAGE * 2 * S.chunk;
    uint64_t *wbar = bars + warp * NSTAGE;
    const int nw = (b1 - b0 - warp + kWarps - 1) / kWarps;  // blocks of this warp (may be <= 0)
    const unsigned char *kc = reinterpret_cast<const unsigned char *>(p.k_cache);
    const unsigned char *vc = reinterpret_cast<const unsigned char *>(p.v_cache);

    auto issue = [&](int j) {
        const int st = j % NSTAGE;
        const int64_t phys = tbl[warp + kWarps * j];
        const int64_t off = ((phys * p.num_kv_heads + kvh) * kBlock) * D * kEsz;
        unsigned char *dst = stages + st * 2 * S.chunk;
        mbar_arrive_expect_tx(&wbar[st], 2 * S.chunk);
        bulk_g2s(dst, kc + off, S.chunk, &wbar[st]);
        bulk_g2s(dst + S.chunk, vc + off, S.chunk, &wbar[st]);
    };
    if (lane == 0)
        for (int j = 0; j < NSTAGE && j < nw; ++j) issue(j);

    SimtState<D, G> state;
    state.init();
    float *pw = p_s + warp * G * kBlock;
    bool ok = true;
    int j = 0;
    for (; j < nw; ++j) {
        const int st = j % NSTAGE;
        // warp-uniform: every lane takes the same branch even if the copy lands
        // just as some lanes give up
        if (!__all_sync(0xffffffffu, mbar_wait(&wbar[st], (j / NSTAGE) & 1))) {
            ok = false;
            break;
        }
        const unsigned char *ks = stages + st * 2 * S.chunk;
        const int base = (b0 + warp + kWarps * j) * kBlock;
        simt_block<T, KT, D, G, kMasked>(state, ks, ks + S.chunk, min(kBlock, L - base), q_s, pw, lane, base, lo, hi);
        if (lane == 0 && j + NSTAGE < nw) {
            fence_proxy_async_smem();
            issue(j + NSTAGE);
        }
    }
    if (!ok) {
        // A copy never completed (the error word is set).  Every copy issued
        // into this warp's ring and not yet consumed (blocks j .. j + NSTAGE - 1)
        // gets one more bounded chance to land before the CTA exits, so none
        // can still be writing into shared memory afterwards; write nothing.
        if (lane == 0)
            for (int jj = j; jj < j + NSTAGE && jj < nw; ++jj)
                mbar_wait(&wbar[jj % NSTAGE], (jj / NSTAGE) & 1, 200000000ll);
        atomicOr(&fail_s, 1);
    }

    // ---- merge the 4 warp states ------------------------------------------
    __syncthreads();  // every warp is done with its stages; reuse them
    if (fail_s) return;
    float *red_acc = reinterpret_cast<float *>(smem);
    constexpr int kPV = SimtState<D, G>::kPV;
    state.finish();
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
        for (int e = 0; e < kPV; ++e) red_acc[(warp * G + h) * D + lane * kPV + e] = state.acc[h][e];
        if (lane == 0) {
            red_m[warp * G + h] = state.m[h];
            red_l[warp * G + h] = state.l[h];
        }
    }
    __syncthreads();
    for (int i = tid; i < rows * D; i += blockDim.x) {
        const int h = i / D, d = i % D;
        float lse;
        float o = combine_warps<D, G, kWarps>(red_m, red_l, red_acc, h, d, &lse);
        o *= p.v_scale;  // V elements are read unscaled (v_scale = 1 for a plain 16-bit call)
        const int64_t qr = row_of(h);
        if (direct) {
            out[qr * D + d] = E::from_float(o);
        } else {
            const int64_t row = qr * p.max_parts + part;
            p.ws_o[row * D + d] = o;
            if (d == 0) p.ws_lse[row] = lse;
        }
    }
}

// out[row, :] = sum_p 2^(lse_p - M) o_p / sum_p 2^(lse_p - M), M = max_p lse_p,
// over the partitions sequence s actually uses (all -inf: a masked row with
// no position, zero).  A CTA of 4 warps takes `rows_per_cta` consecutive rows
// (query token x head) of sequence s.  A lane holds D / 32 consecutive dims,
// so a warp reads one partition's row of o with one coalesced load, and up
// to kInFlight partitions' loads are issued before the first is used.  With
// few partitions (<= kWarpRowParts) each warp merges whole rows on its own;
// with more, the 4 warps share a row (warp w takes partitions w, w + 4, ...)
// and add their sums in shared memory.
constexpr int kMergeWarps = 4;
constexpr int kInFlight = 8;
constexpr int kWarpRowParts = 8;

template <int D>
struct MergeAcc {
    static constexpr int kV = D / 32;  // dims per lane
    float o[kV];
    float w;  // sum of the weights seen
};

// Weighted sum of partitions first, first + stride, ... < n of one row into
// `a` (lane's dims); M is the row's max lse (finite).
template <int D>
__device__ __forceinline__ void merge_accumulate(MergeAcc<D> &a, const float *lse, const float *o_row, int first,
                                                 int stride, int n, float M, int lane) {
    constexpr int kV = MergeAcc<D>::kV;
    for (int i0 = first; i0 < n; i0 += stride * kInFlight) {
        float w[kInFlight];
        float v[kInFlight][kV];
#pragma unroll
        for (int k = 0; k < kInFlight; ++k) {
            const int i = i0 + k * stride;
            w[k] = 0.f;
#pragma unroll
            for (int e = 0; e < kV; ++e) v[k][e] = 0.f;
            const float li = i < n ? lse[i] : -INFINITY;
            // lse = -inf (no position in that partition, or a partition whose
            // tokens another partial of the same CTA holds) gives weight 0,
            // and its o, possibly never written, is not read
            if (li != -INFINITY) {
                w[k] = exp2f(li - M);
                const float *src = o_row + (int64_t)i * D + lane * kV;
                if constexpr (kV == 4) {
                    const float4 x = *reinterpret_cast<const float4 *>(src);
                    v[k][0] = x.x; v[k][1] = x.y; v[k][2] = x.z; v[k][3] = x.w;
                } else {
                    const float2 x = *reinterpret_cast<const float2 *>(src);
                    v[k][0] = x.x; v[k][1] = x.y;
                }
            }
        }
#pragma unroll
        for (int k = 0; k < kInFlight; ++k) {
            a.w += w[k];
#pragma unroll
            for (int e = 0; e < kV; ++e) a.o[e] = fmaf(w[k], v[k][e], a.o[e]);
        }
    }
}

template <typename T, int D>
__device__ __forceinline__ void merge_store(T *out, int lane, const float *o, float wsum) {
    constexpr int kV = D / 32;
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    if constexpr (kV == 4) {
        const typename Elem<T>::T2 a = {Elem<T>::from_float(o[0] * inv), Elem<T>::from_float(o[1] * inv)};
        const typename Elem<T>::T2 b = {Elem<T>::from_float(o[2] * inv), Elem<T>::from_float(o[3] * inv)};
        uint2 u;
        u.x = *reinterpret_cast<const uint32_t *>(&a);
        u.y = *reinterpret_cast<const uint32_t *>(&b);
        *reinterpret_cast<uint2 *>(out + lane * kV) = u;
    } else {
        const typename Elem<T>::T2 a = {Elem<T>::from_float(o[0] * inv), Elem<T>::from_float(o[1] * inv)};
        *reinterpret_cast<typename Elem<T>::T2 *>(out + lane * kV) = a;
    }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

template <typename T, int D>
__global__ void __launch_bounds__(kMergeWarps * 32) merge_part_kernel(const DecodeParams p, const int rows_per_cta) {
    constexpr int kV = MergeAcc<D>::kV;
    __shared__ float red_o[kMergeWarps][D];
    __shared__ float red_w[kMergeWarps];
    const int s = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_launch_dependents();
    pdl_wait();
    const SeqSplit sp = seq_split(p, s, false);
    const int nparts = sp.nparts;
    if (nparts <= 1) return;  // written directly by the decode kernel
    const int rows = p.q_len * p.num_heads;
    const int r0 = blockIdx.x * rows_per_cta;
    const int r1 = min(r0 + rows_per_cta, rows);
    T *out = reinterpret_cast<T *>(p.out);
    auto row_max = [&](const float *lse) {
        float M = -INFINITY;
        for (int i = lane; i < nparts; i += 32) M = fmaxf(M, lse[i]);
        return warp_max(M);
    };
    if (nparts <= kWarpRowParts) {
        // a warp per row
        for (int r = r0 + warp; r < r1; r += kMergeWarps) {
            const int64_t qr = (int64_t)s * rows + r;
            const float *lse = p.ws_lse + qr * p.max_parts;
            const float M = row_max(lse);
            MergeAcc<D> a{};
            if (M != -INFINITY) merge_accumulate<D>(a, lse, p.ws_o + qr * p.max_parts * D, 0, 1, nparts, M, lane);
            merge_store<T, D>(out + qr * D, lane, a.o, a.w);
        }
        return;
    }
    // the CTA's 4 warps per row
    for (int r = r0; r < r1; ++r) {
        const int64_t qr = (int64_t)s * rows + r;
        const float *lse = p.ws_lse + qr * p.max_parts;
        const float M = row_max(lse);
        MergeAcc<D> a{};
        if (M != -INFINITY)
            merge_accumulate<D>(a, lse, p.ws_o + qr * p.max_parts * D, warp, kMergeWarps, nparts, M, lane);
#pragma unroll
        for (int e = 0; e < kV; ++e) red_o[warp][lane * kV + e] = a.o[e];
        if (lane == 0) red_w[warp] = a.w;
        __syncthreads();
        if (warp == 0) {
            float o[kV];
#pragma unroll
            for (int e = 0; e < kV; ++e) {
                o[e] = 0.f;
#pragma unroll
                for (int w = 0; w < kMergeWarps; ++w) o[e] += red_o[w][lane * kV + e];
            }
            float wsum = 0.f;
#pragma unroll
            for (int w = 0; w < kMergeWarps; ++w) wsum += red_w[w];
            merge_store<T, D>(out + qr * D, lane, o, wsum);
        }
        __syncthreads();
    }
}

template <typename T, typename KT, int D, int G, bool kMasked>
cudaError_t launch_part_m(const DecodeParams &p, cudaStream_t stream) {
    constexpr int kEsz = std::is_same<KT, E4M3>::value ? 1 : 2;
    constexpr int kStages = part_stages(G, kEsz);
    auto kern = decode_part_kernel<T, KT, D, G, kStages, kMasked>;
    const int smem = PartLayout(D, G, kStages, kEsz).bytes(p.part_blocks);
    static FuncAttrCache attrs;
    cudaError_t e = ensure_smem(kern, smem, attrs);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, dim3(p.max_parts, p.num_kv_heads, p.num_seqs), dim3(kWarps * 32), smem, stream, p);
    if (e != cudaSuccess || p.max_parts == 1) return e;
    return launch_merge_partitions(p, std::is_same<T, __nv_bfloat16>::value ? PA_BF16 : PA_F16, D, stream);
}

template <typename T, typename KT, int D, int G>
cudaError_t launch_part_t(const DecodeParams &p, cudaStream_t stream) {
    return decode_masked(p) ? launch_part_m<T, KT, D, G, true>(p, stream)
                            : launch_part_m<T, KT, D, G, false>(p, stream);
}

template <typename T, typename KT, int D>
cudaError_t launch_part_d(const DecodeParams &p, int group, cudaStream_t stream) {
    switch (group) {
        case 1: return launch_part_t<T, KT, D, 1>(p, stream);
        case 2: return launch_part_t<T, KT, D, 2>(p, stream);
        case 4: return launch_part_t<T, KT, D, 4>(p, stream);
        case 8: return launch_part_t<T, KT, D, 8>(p, stream);
        case 16: return launch_part_t<T, KT, D, 16>(p, stream);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T, typename KT>
cudaError_t launch_part_k(const DecodeParams &p, int head_dim, int group, cudaStream_t stream) {
    return head_dim == 64 ? launch_part_d<T, KT, 64>(p, group, stream) : launch_part_d<T, KT, 128>(p, group, stream);
}

}  // namespace

cudaError_t launch_merge_partitions(const DecodeParams &p, int dtype, int head_dim, cudaStream_t stream) {
    // Rows per CTA: with few partitions a warp merges a row on its own, so a
    // CTA takes 4 rows (up to 16 for batches with many rows, e.g. several
    // query tokens); with many partitions the 4 warps share a row and a CTA
    // takes 1 row (up to 8 for very large batches).
    const int64_t rows = (int64_t)p.num_heads * p.q_len;
    const int64_t total = rows * p.num_seqs;
    int rpc = 1;
    if (p.max_parts <= kWarpRowParts) {
        rpc = kMergeWarps;
        while (rpc < 16 && total / (rpc * 2) >= 4096) rpc *= 2;
    } else {
        while (rpc < 8 && total / (rpc * 2) >= 8192) rpc *= 2;
    }
    const dim3 grid((unsigned)((rows + rpc - 1) / rpc), p.num_seqs);
    const dim3 block(kMergeWarps * 32);
    if (dtype == PA_F16)
        return head_dim == 64 ? launch_pdl(merge_part_kernel<__half, 64>, grid, block, 0, stream, p, rpc)
                              : launch_pdl(merge_part_kernel<__half, 128>, grid, block, 0, stream, p, rpc);
    return head_dim == 64 ? launch_pdl(merge_part_kernel<__nv_bfloat16, 64>, grid, block, 0, stream, p, rpc)
                          : launch_pdl(merge_part_kernel<__nv_bfloat16, 128>, grid, block, 0, stream, p, rpc);
}

cudaError_t launch_decode_partitioned(const DecodeParams &p, int dtype, int head_dim, int rows, bool fp8_cache,
                                      cudaStream_t stream) {
    if (dtype == PA_F16)
        return fp8_cache ? launch_part_k<__half, E4M3>(p, head_dim, rows, stream)
                         : launch_part_k<__half, __half>(p, head_dim, rows, stream);
    return fp8_cache ? launch_part_k<__nv_bfloat16, E4M3>(p, head_dim, rows, stream)
                     : launch_part_k<__nv_bfloat16, __nv_bfloat16>(p, head_dim, rows, stream);
}

}  // namespace pa
