// pa_cache.cu -- the two companion kernels of paged decode:
//
// reshape_and_cache: "vLLM PagedAttention 大模型推理架构深度实战" section 六,
//   decode loop step "write into the KV cache block": token t's key/value
//   rows go to slot slot_mapping[t] = block * 16 + offset of the head-major
//   pool [NB, Hk, 16, D].
// copy_blocks: same page, section 2.3: a block shared by several sequences is
//   copied before one of them writes into it (copy-on-write).
// swap_blocks: same page, section 3.2 (a preempted sequence's KV cache is
//   swapped out to CPU memory and swapped back in on resume) and section 九
//   item 5 (swapped-out KV kept in fast host memory): block copies between a
//   device pool and a page-locked host pool, which the kernel reads or writes
//   directly through unified addressing (one launch for all pairs).
//
// Both are pure data movement (bit-exact) and HBM-bound: 16-byte vector
// loads and stores, consecutive threads on consecutive 16-byte chunks.
#include "pa_common.cuh"
#include "pa_decode.h"

namespace pa {

__device__ unsigned int g_device_error = 0;

namespace {

constexpr int kBlock = 16;
constexpr int kCopyLayers = 64;  // layer pointers per copy_blocks launch

// One thread per 16-byte chunk of a (token, kv head) row, for key and value.
__global__ void __launch_bounds__(256)
    reshape_and_cache_kernel(const uint4 *__restrict__ key, const uint4 *__restrict__ value,
                             uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache,
                             const int64_t *__restrict__ slot_mapping, int64_t num_items, int chunks_per_row,
                             int num_kv_heads, int64_t num_slots) {
    pdl_launch_dependents();
    pdl_wait();
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= num_items) return;
    const int64_t row = i / chunks_per_row;  // (token, kv head)
    const int c = (int)(i % chunks_per_row);
    const int64_t t = row / num_kv_heads;
    const int h = (int)(row % num_kv_heads);
    const int64_t slot = slot_mapping[t];
    if (slot < 0) return;  // padding token
    if (slot >= num_slots) {
        if (h == 0 && c == 0) flag_error(PA_DEVERR_SLOT);
        return;
    }
    const int64_t blk = slot / kBlock, off = slot % kBlock;
    const int64_t dst = ((blk * num_kv_heads + h) * kBlock + off) * chunks_per_row + c;
    k_cache[dst] = key[i];
    v_cache[dst] = value[i];
}

struct LayerPtrs {
    uint4 *k[kCopyLayers];
    uint4 *v[kCopyLayers];
};

// CTA = (pair, layer): copies the whole K block and V block.
__global__ void __launch_bounds__(256)
    copy_blocks_kernel(const LayerPtrs ptrs, const int64_t *__restrict__ block_mapping, int64_t chunks_per_block,
                       int64_t num_blocks) {
    pdl_launch_dependents();
    pdl_wait();
    const int pair = blockIdx.x, layer = blockIdx.y;
    const int64_t src = block_mapping[2 * pair], dst = block_mapping[2 * pair + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (threadIdx.x == 0 && layer == 0) flag_error(PA_DEVERR_COPY_PAIR);
        return;
    }
    const uint4 *ks = ptrs.k[layer] + src * chunks_per_block;
    const uint4 *vs = ptrs.v[layer] + src * chunks_per_block;
    uint4 *kd = ptrs.k[layer] + dst * chunks_per_block;
    uint4 *vd = ptrs.v[layer] + dst * chunks_per_block;
    for (int64_t i = threadIdx.x; i < chunks_per_block; i += blockDim.x) {
        const uint4 a = ks[i];
        const uint4 b = vs[i];
        kd[i] = a;
        vd[i] = b;
    }
}

// CTA = (pair, K or V): copies one block between the two pools.  Each thread
// keeps 4 16-byte loads in flight before storing, since host-side accesses
// cross the PCIe / chip-to-chip link with a long latency.
__global__ void __launch_bounds__(256)
    swap_blocks_kernel(const uint4 *__restrict__ src_k, const uint4 *__restrict__ src_v, int64_t src_blocks,
                       uint4 *__restrict__ dst_k, uint4 *__restrict__ dst_v, int64_t dst_blocks,
                       const int64_t *__restrict__ block_mapping, int64_t chunks_per_block) {
    pdl_launch_dependents();
    pdl_wait();
    const int pair = blockIdx.x;
    const int64_t src = block_mapping[2 * pair], dst = block_mapping[2 * pair + 1];
    if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
        if (threadIdx.x == 0 && blockIdx.y == 0) flag_error(PA_DEVERR_COPY_PAIR);
        return;
    }
    const uint4 *s = (blockIdx.y == 0 ? src_k : src_v) + src * chunks_per_block;
    uint4 *d = (blockIdx.y == 0 ? dst_k : dst_v) + dst * chunks_per_block;
    constexpr int kUnroll = 4;
    for (int64_t i0 = threadIdx.x; i0 < chunks_per_block; i0 += (int64_t)blockDim.x * kUnroll) {
        uint4 r[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = i0 + (int64_t)u * blockDim.x;
            if (i < chunks_per_block) r[u] = s[i];
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = i0 + (int64_t)u * blockDim.x;
            if (i < chunks_per_block) d[i] = r[u];
        }
    }
}

// One thread per 16 elements of a (token, kv head) row: two 16-byte loads of
// key (value), a correctly rounded fp32 division by the tensor's scale, then
// round-to-nearest-even to E4M3 with saturation, one 16-byte store.
template <typename T>
__global__ void __launch_bounds__(256)
    reshape_and_cache_fp8_kernel(const T *__restrict__ key, const T *__restrict__ value, uint8_t *__restrict__ k_cache,
                                 uint8_t *__restrict__ v_cache, const int64_t *__restrict__ slot_mapping,
                                 int64_t num_items, int items_per_row, int head_dim, int num_kv_heads,
                                 int64_t num_slots, float k_scale, float v_scale) {
    pdl_launch_dependents();
    pdl_wait();
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= num_items) return;
    const int64_t row = i / items_per_row;  // (token, kv head)
    const int c = (int)(i % items_per_row);
    const int64_t t = row / num_kv_heads;
    const int h = (int)(row % num_kv_heads);
    const int64_t slot = slot_mapping[t];
    if (slot < 0) return;
    if (slot >= num_slots) {
        if (h == 0 && c == 0) flag_error(PA_DEVERR_SLOT);
        return;
    }
    const int64_t blk = slot / kBlock, off = slot % kBlock;
    const int64_t dst = ((blk * num_kv_heads + h) * kBlock + off) * head_dim + c * 16;
    auto quantize16 = [&](const T *src, float sc, uint8_t *out) {
        const uint4 a = reinterpret_cast<const uint4 *>(src)[0];
        const uint4 b = reinterpret_cast<const uint4 *>(src)[1];
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint32_t packed[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 x0 = Elem<T>::to_float2(w[2 * j]);
            const float2 x1 = Elem<T>::to_float2(w[2 * j + 1]);
            const uint16_t lo = float2_to_e4m3x2(__fdiv_rn(x0.x, sc), __fdiv_rn(x0.y, sc));
            const uint16_t hi = float2_to_e4m3x2(__fdiv_rn(x1.x, sc), __fdiv_rn(x1.y, sc));
            packed[j] = (uint32_t)lo | ((uint32_t)hi << 16);
        }
        *reinterpret_cast<uint4 *>(out) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    };
    const int64_t src = row * head_dim + c * 16;
    quantize16(key + src, k_scale, k_cache + dst);
    quantize16(value + src, v_scale, v_cache + dst);
}

// Diagnostic: one thread waits on an mbarrier that nothing ever arrives on,
// with a bound of `limit_cycles` SM cycles; the bounded wait gives up, sets
// PA_DEVERR_TIMEOUT and the kernel returns.  The same wait (with its longer
// default bound) guards every pipeline stage of the decode kernels.
__global__ void wait_timeout_probe_kernel(long long limit_cycles) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait(&bar, 0, limit_cycles);  // never completes: no arrival
}

}  // namespace

cudaError_t launch_wait_timeout_probe(long long limit_cycles, cudaStream_t stream) {
    wait_timeout_probe_kernel<<<1, 32, 0, stream>>>(limit_cycles);
    return cudaGetLastError();
}

cudaError_t launch_reshape_and_cache_fp8(const void *key, const void *value, void *k_cache, void *v_cache,
                                         const int64_t *slot_mapping, int32_t num_tokens, const CacheDims &d,
                                         int dtype, float k_scale, float v_scale, cudaStream_t stream) {
    const int ipr = d.head_dim / 16;
    const int64_t items = (int64_t)num_tokens * d.num_kv_heads * ipr;
    if (items == 0) return cudaSuccess;
    const dim3 grid((unsigned)((items + 255) / 256));
    const int64_t slots = (int64_t)d.num_blocks * kBlock;
    uint8_t *kc = static_cast<uint8_t *>(k_cache), *vc = static_cast<uint8_t *>(v_cache);
    if (dtype == PA_F16)
        return launch_pdl(reshape_and_cache_fp8_kernel<__half>, grid, dim3(256), 0, stream,
                          static_cast<const __half *>(key), static_cast<const __half *>(value), kc, vc, slot_mapping,
                          items, ipr, (int)d.head_dim, (int)d.num_kv_heads, slots, k_scale, v_scale);
    return launch_pdl(reshape_and_cache_fp8_kernel<__nv_bfloat16>, grid, dim3(256), 0, stream,
                      static_cast<const __nv_bfloat16 *>(key), static_cast<const __nv_bfloat16 *>(value), kc, vc,
                      slot_mapping, items, ipr, (int)d.head_dim, (int)d.num_kv_heads, slots, k_scale, v_scale);
}

cudaError_t launch_swap_blocks(const void *src_k, const void *src_v, int64_t src_blocks, void *dst_k, void *dst_v,
                               int64_t dst_blocks, const int64_t *block_mapping, int32_t num_pairs, const CacheDims &d,
                               cudaStream_t stream) {
    if (num_pairs == 0) return cudaSuccess;
    const int64_t chunks = (int64_t)d.num_kv_heads * kBlock * d.head_dim * d.elem_bytes / 16;
    return launch_pdl(swap_blocks_kernel, dim3(num_pairs, 2), dim3(256), 0, stream, static_cast<const uint4 *>(src_k),
                      static_cast<const uint4 *>(src_v), src_blocks, static_cast<uint4 *>(dst_k),
                      static_cast<uint4 *>(dst_v), dst_blocks, block_mapping, chunks);
}

cudaError_t launch_reshape_and_cache(const void *key, const void *value, void *k_cache, void *v_cache,
                                     const int64_t *slot_mapping, int32_t num_tokens, const CacheDims &d,
                                     cudaStream_t stream) {
    const int chunks = d.head_dim / 8;
    const int64_t items = (int64_t)num_tokens * d.num_kv_heads * chunks;
    if (items == 0) return cudaSuccess;
    const int64_t grid = (items + 255) / 256;
    return launch_pdl(reshape_and_cache_kernel, dim3((unsigned)grid), dim3(256), 0, stream,
                      static_cast<const uint4 *>(key), static_cast<const uint4 *>(value), static_cast<uint4 *>(k_cache),
                      static_cast<uint4 *>(v_cache), slot_mapping, items, chunks, (int)d.num_kv_heads,
                      (int64_t)d.num_blocks * kBlock);
}

cudaError_t launch_copy_blocks(void *const *k_caches, void *const *v_caches, int32_t num_layers,
                               const int64_t *block_mapping, int32_t num_pairs, const CacheDims &d,
                               cudaStream_t stream) {
    if (num_pairs == 0 || num_layers == 0) return cudaSuccess;
    const int64_t chunks = (int64_t)d.num_kv_heads * kBlock * d.head_dim * d.elem_bytes / 16;
    for (int l0 = 0; l0 < num_layers; l0 += kCopyLayers) {
        const int nl = num_layers - l0 < kCopyLayers ? num_layers - l0 : kCopyLayers;
        LayerPtrs ptrs = {};
        for (int i = 0; i < nl; ++i) {
            ptrs.k[i] = static_cast<uint4 *>(k_caches[l0 + i]);
            ptrs.v[i] = static_cast<uint4 *>(v_caches[l0 + i]);
        }
        cudaError_t e = launch_pdl(copy_blocks_kernel, dim3(num_pairs, nl), dim3(256), 0, stream, ptrs, block_mapping,
                                   chunks, (int64_t)d.num_blocks);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace pa
