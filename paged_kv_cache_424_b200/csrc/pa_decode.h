// pa_decode.h -- private interface between the C ABI (pa_api.cu) and the
// kernel launchers.  Not installed; the public interface is include/pa.h.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/pa.h"

namespace pa {

constexpr int kMaxDevices = 64;

// Everything a decode launch needs; passed by value as the kernel argument.
struct DecodeParams {
    void *out;                   // [S, H, D] fp16/bf16
    const void *q;               // [S, H, D]
    const void *k_cache;         // [NB, Hk, 16, D]
    const void *v_cache;         // [NB, Hk, 16, D]
    const int32_t *block_tables; // [S, MB]
    const int32_t *context_lens; // [S]
    float *ws_o;                 // [S, H, max_parts, D] partial outputs (split only)
    float *ws_lse;               // [S, H, max_parts] log2-sum-exp per partial
    float scale_log2;            // scale * log2(e) (times k_scale for an FP8 cache)
    float v_scale;               // applied to the output (1 unless the cache is FP8)
    int32_t num_seqs, num_heads, num_kv_heads, max_blocks_per_seq;
    int64_t num_blocks;
    int32_t part_blocks;         // table entries per KV partition
    int32_t max_parts;           // partitions in the grid (gridDim.x)
    int32_t group;               // query heads per KV head
    int32_t q_len;               // query tokens per sequence (q, out: [S, q_len, H, D])
    int32_t window;              // sliding window in tokens, 0 = none
    const int32_t *seq_order;    // nullptr, or the sequence each blockIdx.z visits
    int32_t parts_per_cta;       // tensor-core kernel: consecutive partitions one CTA streams (1 elsewhere)
    int32_t heads_per_cta;       // tensor-core kernel, plain decode: consecutive KV heads one CTA streams (1 elsewhere)
    int32_t part_major;          // tensor-core kernel: grid (head, position, partition) instead of (partition, head, position)
};

// Whether a launch needs per-row position masks (several query tokens or a
// sliding window); the kernels take this as a template flag.
inline bool decode_masked(const DecodeParams &p) { return p.q_len != 1 || p.window != 0; }

// Per-device record of the function attributes a kernel has been given
// (one per kernel instantiation).  Launches may come from several host
// threads: the fast path is one atomic load, and the attribute calls run
// under a lock so the recorded value never exceeds what was really set.
struct FuncAttrCache {
    std::atomic<int> smem[kMaxDevices] = {};      // dynamic shared-memory limit set
    std::atomic<int> carveout[kMaxDevices] = {};  // 1 once the carveout preference is set
    std::mutex mu;
};

// Raise a kernel's dynamic shared-memory limit on the current device when a
// launch needs more than was set before (the attribute is per device), and
// optionally ask for the largest shared-memory carveout once.
template <typename K>
inline cudaError_t ensure_smem(K kern, int bytes, FuncAttrCache &cache, bool max_carveout = false) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    const bool need_smem = bytes > 48 * 1024 && bytes > cache.smem[dev].load(std::memory_order_acquire);
    const bool need_carveout = max_carveout && !cache.carveout[dev].load(std::memory_order_acquire);
    if (!need_smem && !need_carveout) return cudaSuccess;
    std::lock_guard<std::mutex> lock(cache.mu);
    if (max_carveout && !cache.carveout[dev].load(std::memory_order_relaxed)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        cache.carveout[dev].store(1, std::memory_order_release);
    }
    if (bytes > 48 * 1024 && bytes > cache.smem[dev].load(std::memory_order_relaxed)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e != cudaSuccess) return e;
        cache.smem[dev].store(bytes, std::memory_order_release);
    }
    return cudaSuccess;
}

// Record `msg` as the text pa_last_error() returns on this thread; returns st.
pa_status set_last_error(pa_status st, const char *msg);

// Fixed-partition decode (+ merge when max_parts > 1) on `stream`; the
// caches hold elements of `dtype`, or FP8 E4M3 codes when `fp8_cache`.
// `rows` is the row capacity per KV head (1, 2, 4, 8 or 16 >= group * q_len).
cudaError_t launch_decode_partitioned(const DecodeParams &p, int dtype, int head_dim, int rows, bool fp8_cache,
                                      cudaStream_t stream);


// Log-sum-exp merge of the partitions written to the workspace.
cudaError_t launch_merge_partitions(const DecodeParams &p, int dtype, int head_dim, cudaStream_t stream);

// Tensor-core decode for row capacities 4, 8 or 16 at head_dim 128 (GQA
// groups, or several query tokens) and whether it applies to these sizes.
bool decode_tc_supported(int head_dim, int rows, int64_t num_blocks, int num_kv_heads);
cudaError_t launch_decode_tc(const DecodeParams &p, int dtype, int rows, bool fp8_cache, cudaStream_t stream);

// Cache kernels.
struct CacheDims {
    int32_t num_kv_heads, head_dim;
    int64_t num_blocks;
    int32_t elem_bytes;  // 2 for fp16 / bf16, 1 for FP8 E4M3
};
cudaError_t launch_reshape_and_cache(const void *key, const void *value, void *k_cache, void *v_cache,
                                     const int64_t *slot_mapping, int32_t num_tokens, const CacheDims &d,
                                     cudaStream_t stream);
cudaError_t launch_reshape_and_cache_fp8(const void *key, const void *value, void *k_cache, void *v_cache,
                                         const int64_t *slot_mapping, int32_t num_tokens, const CacheDims &d,
                                         int dtype, float k_scale, float v_scale, cudaStream_t stream);
cudaError_t launch_copy_blocks(void *const *k_caches, void *const *v_caches, int32_t num_layers,
                               const int64_t *block_mapping, int32_t num_pairs, const CacheDims &d,
                               cudaStream_t stream);
cudaError_t launch_wait_timeout_probe(long long limit_cycles, cudaStream_t stream);
cudaError_t launch_swap_blocks(const void *src_k, const void *src_v, int64_t src_blocks, void *dst_k, void *dst_v,
                               int64_t dst_blocks, const int64_t *block_mapping, int32_t num_pairs, const CacheDims &d,
                               cudaStream_t stream);

}  // namespace pa
