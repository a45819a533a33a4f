// pa_decode.cu -- paged decode attention, CUDA-core path, and the split-KV
// log-sum-exp merge.
//
// Method: "vLLM PagedAttention 大模型推理架构深度实战" section 2.2 (a sequence's
// KV lives in 16-token physical blocks named by its block table) and section
// 5.1 (exact attention, blocks combined by online softmax);
// "vLLM：重塑大模型推理性能的关键引擎", PagedAttention section, kernel sketch
// (ceil(len / 16) blocks, entry i of the table row is logical block i).
//
// Work decomposition (B200: 148 SMs, HBM-bound):
//   CTA = (KV partition p, KV head kvh, sequence s), 4 warps.  The CTA's
//   partition covers table entries [p * part_blocks, ...).  Warp w takes
//   the partition's blocks w, w + 4, w + 8, ... and streams them through its
//   own NSTAGE-deep ring of shared-memory stages: one lane issues two 1-D
//   bulk copies (the K chunk and the V chunk of (block, kvh), each one
//   contiguous 16 x D x 2-byte run in the head-major pool) that complete on
//   the stage's mbarrier.  Each warp keeps an online-softmax state
//   (running max m, running sum l, accumulator) for the G query heads that
//   share kvh; at the end the 4 warp states are merged in shared memory.
//   If the sequence needs one partition the CTA writes the output;
//   otherwise it writes (o_p, log2-sum-exp_p) to the workspace and the merge
//   kernel combines partitions:  out = sum_p 2^(lse_p - M) o_p / sum_p 2^(lse_p - M).
//
// Logits are kept in the log2 domain: q is pre-scaled by scale * log2(e),
// so softmax weights are exp2(x - m).
#include "pa_common.cuh"
#include "pa_decode.h"

namespace pa {

namespace {

constexpr int kBlock = 16;  // tokens per KV block
constexpr int kWarps = 4;

__device__ __forceinline__ float fast_exp2(float x) { return exp2f(x); }

// Context length of sequence s, checked against the table row and the
// partition grid; out-of-range values are clamped and flagged.
__device__ __forceinline__ int checked_len(const DecodeParams &p, int s, bool report) {
    int L = p.context_lens[s];
    const int lmax = min(p.max_blocks_per_seq * kBlock, p.max_parts * p.part_blocks * kBlock);
    if (L < 0 || L > lmax) {
        if (report) flag_error(PA_DEVERR_CONTEXT);
        L = L < 0 ? 0 : lmax;
    }
    return L;
}

// Shared-memory layout of the CUDA-core kernel (bytes):
//   [main]  per-warp stage rings (kWarps x NSTAGE x {K chunk, V chunk}); reused
//           at the end for the cross-warp reduction (kWarps x G x D floats)
//   [q]     G x 2 halves x (D/16 chunks x 12 floats)  (padded query rows)
//   [p]     kWarps x G x 16 floats                     (softmax weights)
//   [m, l]  2 x kWarps x G floats
//   [bars]  kWarps x NSTAGE mbarriers
//   [table] part_blocks int32
struct SimtLayout {
    int chunk, qhalf, main, q_off, p_off, ml_off, bar_off, table_off;
    __host__ __device__ constexpr SimtLayout(int D, int G, int nstage)
        : chunk(kBlock * D * 2), qhalf((D / 16) * 12),
          main(kWarps * nstage * 2 * kBlock * D * 2 > kWarps * G * D * 4 ? kWarps * nstage * 2 * kBlock * D * 2
                                                                        : kWarps * G * D * 4),
          q_off(main), p_off(q_off + G * 2 * (D / 16) * 12 * 4), ml_off(p_off + kWarps * G * kBlock * 4),
          bar_off((ml_off + 2 * kWarps * G * 4 + 7) / 8 * 8), table_off(bar_off + kWarps * nstage * 8) {}
    __host__ __device__ constexpr int bytes(int part_blocks) const { return table_off + part_blocks * 4; }
};

constexpr int kSimtStages = 3;

template <typename T, int D, int G, int NSTAGE>
__global__ void __launch_bounds__(kWarps * 32)
    decode_simt_kernel(const DecodeParams p) {
    constexpr SimtLayout S(D, G, NSTAGE);
    using E = Elem<T>;
    constexpr int kNC = D / 16;
    constexpr int kPV = D / 32;  // output dims per lane

    extern __shared__ __align__(128) unsigned char smem[];
    float *q_s = reinterpret_cast<float *>(smem + S.q_off);
    float *p_s = reinterpret_cast<float *>(smem + S.p_off);
    float *red_m = reinterpret_cast<float *>(smem + S.ml_off);
    float *red_l = red_m + kWarps * G;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S.bar_off);
    int32_t *tbl = reinterpret_cast<int32_t *>(smem + S.table_off);
    __shared__ int fail_s;

    const int part = blockIdx.x, kvh = blockIdx.y, s = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.num_heads;
    const int head0 = kvh * G;

    const int L = checked_len(p, s, part == 0 && kvh == 0 && tid == 0);
    const int nblk = (L + kBlock - 1) / kBlock;
    const int nparts = nblk == 0 ? 1 : (nblk + p.part_blocks - 1) / p.part_blocks;
    if (part >= nparts) return;
    const bool direct = nparts == 1;
    T *out = reinterpret_cast<T *>(p.out);

    if (L == 0) {  // empty context: zero rows
        for (int i = tid; i < G * D; i += blockDim.x)
            out[((int64_t)s * H + head0 + i / D) * D + i % D] = E::from_float(0.f);
        return;
    }

    const int b0 = part * p.part_blocks;
    const int b1 = min(b0 + p.part_blocks, nblk);

    // Block-table slice -> shared memory (range-checked).
    for (int i = tid; i < b1 - b0; i += blockDim.x) {
        int b = p.block_tables[(int64_t)s * p.max_blocks_per_seq + b0 + i];
        if (b < 0 || (int64_t)b >= p.num_blocks) {
            flag_error(PA_DEVERR_BLOCK_ID);
            b = 0;
        }
        tbl[i] = b;
    }
    // Query rows of the group, scaled into the log2 domain, in a padded
    // layout [h][half][chunk][12] that keeps the rotated reads conflict-free.
    {
        const T *q = reinterpret_cast<const T *>(p.q) + ((int64_t)s * H + head0) * D;
        for (int i = tid; i < G * D / 2; i += blockDim.x) {
            const int h = i / (D / 2), e2 = (i % (D / 2)) * 2;
            const uint32_t bits = *reinterpret_cast<const uint32_t *>(q + h * D + e2);
            const float2 f = E::to_float2(bits);
            const int half = e2 / (D / 2), e = e2 % (D / 2);
            float *dst = q_s + (h * 2 + half) * S.qhalf + (e / 8) * 12 + (e % 8);
            dst[0] = f.x * p.scale_log2;
            dst[1] = f.y * p.scale_log2;
        }
    }
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
    const T *kc = reinterpret_cast<const T *>(p.k_cache);
    const T *vc = reinterpret_cast<const T *>(p.v_cache);

    auto issue = [&](int j) {
        const int st = j % NSTAGE;
        const int64_t phys = tbl[warp + kWarps * j];
        const int64_t off = ((phys * p.num_kv_heads + kvh) * kBlock) * D;
        unsigned char *dst = stages + st * 2 * S.chunk;
        mbar_arrive_expect_tx(&wbar[st], 2 * S.chunk);
        bulk_g2s(dst, kc + off, S.chunk, &wbar[st]);
        bulk_g2s(dst + S.chunk, vc + off, S.chunk, &wbar[st]);
    };
    if (lane == 0)
        for (int j = 0; j < NSTAGE && j < nw; ++j) issue(j);

    float m[G], l[G], acc[G][kPV];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
#pragma unroll
        for (int e = 0; e < kPV; ++e) acc[h][e] = 0.f;
    }

    const int t = lane >> 1, half = lane & 1;
    float *pw = p_s + warp * G * kBlock;
    bool ok = true;
    for (int j = 0; j < nw; ++j) {
        const int st = j % NSTAGE;
        if (!mbar_wait(&wbar[st], (j / NSTAGE) & 1)) {
            ok = false;
            break;
        }
        const unsigned char *ks = stages + st * 2 * S.chunk;
        const unsigned char *vs = ks + S.chunk;
        const int base = (b0 + warp + kWarps * j) * kBlock;
        const int nvalid = min(kBlock, L - base);

        // logits: lane pair (2t, 2t+1) splits token t's D dims in halves
        float x[G];
#pragma unroll
        for (int h = 0; h < G; ++h) x[h] = 0.f;
        const unsigned char *krow = ks + t * D * 2 + half * D;
#pragma unroll
        for (int i = 0; i < kNC; ++i) {
            const int c = (i + lane) & (kNC - 1);
            const uint4 raw = *reinterpret_cast<const uint4 *>(krow + c * 16);
            const float2 k0 = E::to_float2(raw.x), k1 = E::to_float2(raw.y);
            const float2 k2 = E::to_float2(raw.z), k3 = E::to_float2(raw.w);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float *qc = q_s + (h * 2 + half) * S.qhalf + c * 12;
                const float4 qa = *reinterpret_cast<const float4 *>(qc);
                const float4 qb = *reinterpret_cast<const float4 *>(qc + 4);
                float a = x[h];
                a = fmaf(k0.x, qa.x, a);
                a = fmaf(k0.y, qa.y, a);
                a = fmaf(k1.x, qa.z, a);
                a = fmaf(k1.y, qa.w, a);
                a = fmaf(k2.x, qb.x, a);
                a = fmaf(k2.y, qb.y, a);
                a = fmaf(k3.x, qb.z, a);
                a = fmaf(k3.y, qb.w, a);
                x[h] = a;
            }
        }
        float alpha[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float v = x[h] + __shfl_xor_sync(0xffffffffu, x[h], 1);
            v = (t < nvalid) ? v : -INFINITY;
            float bm = v;
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
            const float mn = fmaxf(m[h], bm);
            const float pr = fast_exp2(v - mn);
            float ps = pr;
            ps += __shfl_xor_sync(0xffffffffu, ps, 2);
            ps += __shfl_xor_sync(0xffffffffu, ps, 4);
            ps += __shfl_xor_sync(0xffffffffu, ps, 8);
            ps += __shfl_xor_sync(0xffffffffu, ps, 16);
            alpha[h] = fast_exp2(m[h] - mn);
            l[h] = l[h] * alpha[h] + ps;
            m[h] = mn;
            if (half == 0) pw[h * kBlock + t] = pr;
        }
        __syncwarp();

        // P V: lane owns dims [lane * kPV, lane * kPV + kPV)
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < kPV; ++e) acc[h][e] *= alpha[h];
#pragma unroll
        for (int tq = 0; tq < kBlock / 4; ++tq) {
            if (tq * 4 < nvalid) {
                float4 pq[G];
#pragma unroll
                for (int h = 0; h < G; ++h) pq[h] = *reinterpret_cast<const float4 *>(pw + h * kBlock + tq * 4);
#pragma unroll
                for (int tt = 0; tt < 4; ++tt) {
                    const int tok = tq * 4 + tt;
                    if (tok < nvalid) {
                        float vf[kPV];
                        if constexpr (kPV == 4) {
                            const uint2 raw = *reinterpret_cast<const uint2 *>(vs + tok * D * 2 + lane * 8);
                            const float2 a = E::to_float2(raw.x), b = E::to_float2(raw.y);
                            vf[0] = a.x; vf[1] = a.y; vf[2] = b.x; vf[3] = b.y;
                        } else {
                            const uint32_t raw = *reinterpret_cast<const uint32_t *>(vs + tok * D * 2 + lane * 4);
                            const float2 a = E::to_float2(raw);
                            vf[0] = a.x; vf[1] = a.y;
                        }
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            const float pv = tt == 0 ? pq[h].x : tt == 1 ? pq[h].y : tt == 2 ? pq[h].z : pq[h].w;
#pragma unroll
                            for (int e = 0; e < kPV; ++e) acc[h][e] = fmaf(pv, vf[e], acc[h][e]);
                        }
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0 && j + NSTAGE < nw) {
            fence_proxy_async_smem();
            issue(j + NSTAGE);
        }
    }
    if (!ok) {
        // A copy never completed (the error word is set).  Give it one more
        // bounded chance to land before the CTA exits; write nothing.
        if (lane == 0) mbar_wait(&wbar[0], 0, 100000000ull);
        atomicOr(&fail_s, 1);
    }

    // ---- merge the 4 warp states ------------------------------------------
    __syncthreads();  // every warp is done with its stages; reuse them
    if (fail_s) return;
    float *red_acc = reinterpret_cast<float *>(smem);
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
        for (int e = 0; e < kPV; ++e) red_acc[(warp * G + h) * D + lane * kPV + e] = acc[h][e];
        if (lane == 0) {
            red_m[warp * G + h] = m[h];
            red_l[warp * G + h] = l[h];
        }
    }
    __syncthreads();
    for (int i = tid; i < G * D; i += blockDim.x) {
        const int h = i / D, d = i % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, red_m[w * G + h]);
        float lsum = 0.f, o = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float f = fast_exp2(red_m[w * G + h] - M);  // 0 for warps without blocks
            lsum = fmaf(red_l[w * G + h], f, lsum);
            o = fmaf(red_acc[(w * G + h) * D + d], f, o);
        }
        const int head = head0 + h;
        if (direct) {
            out[((int64_t)s * H + head) * D + d] = E::from_float(o / lsum);
        } else {
            const int64_t row = ((int64_t)s * H + head) * p.max_parts + part;
            p.ws_o[row * D + d] = o / lsum;
            if (d == 0) p.ws_lse[row] = M + log2f(lsum);
        }
    }
}

// out[s, h, :] = sum_p 2^(lse_p - M) o_p / sum_p 2^(lse_p - M), M = max_p lse_p,
// over the partitions sequence s actually uses.  One CTA of D threads per (h, s).
template <typename T, int D>
__global__ void __launch_bounds__(D) merge_kernel(const DecodeParams p) {
    const int h = blockIdx.x, s = blockIdx.y, d = threadIdx.x;
    const int L = checked_len(p, s, false);
    const int nblk = (L + kBlock - 1) / kBlock;
    const int nparts = (nblk + p.part_blocks - 1) / p.part_blocks;
    if (nparts <= 1) return;  // written directly by the decode kernel
    const int64_t row = ((int64_t)s * p.num_heads + h) * p.max_parts;
    const float *lse = p.ws_lse + row;
    float M = -INFINITY;
    for (int i = 0; i < nparts; ++i) M = fmaxf(M, lse[i]);
    float wsum = 0.f, o = 0.f;
    for (int i = 0; i < nparts; ++i) {
        const float w = exp2f(lse[i] - M);
        wsum += w;
        o = fmaf(w, p.ws_o[(row + i) * D + d], o);
    }
    reinterpret_cast<T *>(p.out)[((int64_t)s * p.num_heads + h) * D + d] = Elem<T>::from_float(o / wsum);
}

// Raise the kernel's dynamic shared-memory limit on the current device when a
// launch needs more than was set before (cudaFuncSetAttribute is per device).
template <typename K>
cudaError_t ensure_smem(K kern, int bytes, int *configured_per_device) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (bytes > 48 * 1024 && bytes > configured_per_device[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e != cudaSuccess) return e;
        configured_per_device[dev] = bytes;
    }
    return cudaSuccess;
}

template <typename T, int D, int G>
cudaError_t launch_simt_t(const DecodeParams &p, cudaStream_t stream) {
    auto kern = decode_simt_kernel<T, D, G, kSimtStages>;
    const int smem = SimtLayout(D, G, kSimtStages).bytes(p.part_blocks);
    static int configured[kMaxDevices] = {};
    cudaError_t e = ensure_smem(kern, smem, configured);
    if (e != cudaSuccess) return e;
    dim3 grid(p.max_parts, p.num_kv_heads, p.num_seqs);
    kern<<<grid, kWarps * 32, smem, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess || p.max_parts == 1) return e;
    merge_kernel<T, D><<<dim3(p.num_heads, p.num_seqs), D, 0, stream>>>(p);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_simt_d(const DecodeParams &p, int group, cudaStream_t stream) {
    switch (group) {
        case 1: return launch_simt_t<T, D, 1>(p, stream);
        case 2: return launch_simt_t<T, D, 2>(p, stream);
        case 4: return launch_simt_t<T, D, 4>(p, stream);
        case 8: return launch_simt_t<T, D, 8>(p, stream);
        case 16: return launch_simt_t<T, D, 16>(p, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

int decode_simt_smem_bytes(int head_dim, int group, int part_blocks) {
    return SimtLayout(head_dim, group, kSimtStages).bytes(part_blocks);
}

cudaError_t launch_decode_simt(const DecodeParams &p, int dtype, int head_dim, int group, cudaStream_t stream) {
    if (dtype == PA_F16)
        return head_dim == 64 ? launch_simt_d<__half, 64>(p, group, stream)
                              : launch_simt_d<__half, 128>(p, group, stream);
    return head_dim == 64 ? launch_simt_d<__nv_bfloat16, 64>(p, group, stream)
                          : launch_simt_d<__nv_bfloat16, 128>(p, group, stream);
}

}  // namespace pa
