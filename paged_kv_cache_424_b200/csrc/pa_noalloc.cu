// pa_noalloc.cu -- pa_decode_noalloc: decode attention whose split-KV scratch
// lives in a fixed device array owned by the library, for callers that
// cannot allocate device memory at call time (see include/pa.h).
//
// The scratch is a file-scope __device__ array of kNoAllocScratchBytes.  Host
// code cannot use the array's name as a device address, so on the first call
// on each device (with that device current) the entry point asks the runtime
// for the array's device address once, checks the result, keeps it, and
// passes it to the existing decode path as its workspace.  Nothing here calls
// cudaMalloc, cudaFree or any allocating library routine.
#include <cstdio>
#include <mutex>

#include "../../include/pa.h"
#include "pa_decode.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB per device

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mu;
void *g_scratch_addr[pa::kMaxDevices] = {};

// Device address of the scratch array on the current device (set-up on the
// first call per device).
pa_status scratch_address(void **addr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return pa::set_last_error(PA_ERR_CUDA, "pa_decode_noalloc: cudaGetDevice failed");
    if (dev < 0 || dev >= pa::kMaxDevices)
        return pa::set_last_error(PA_ERR_CUDA, "pa_decode_noalloc: device ordinal out of range");
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return pa::set_last_error(PA_ERR_CUDA, "pa_decode_noalloc: cudaGetSymbolAddress of the scratch failed");
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_noalloc(void *out, const void *q, const void *k_cache, const void *v_cache,
                                       const int32_t *block_tables, const int32_t *context_lens, float scale,
                                       int32_t num_kv_heads, const pa_dims *dims, int32_t max_context_len,
                                       int32_t partition_tokens, void *stream) {
    const int32_t parts = pa_decode_num_partitions(dims, max_context_len, partition_tokens);
    if (parts < 0) return static_cast<pa_status>(parts);
    const size_t need = pa_decode_workspace_size(dims, max_context_len, partition_tokens);
    if (need > kNoAllocScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "pa_decode_noalloc: this call needs %zu bytes of split-KV scratch but the library's static "
                 "scratch holds %zu; use pa_decode with a caller workspace, larger partitions or fewer sequences",
                 need, kNoAllocScratchBytes);
        return pa::set_last_error(PA_ERR_WORKSPACE, msg);
    }
    void *scratch = nullptr;
    if (need > 0) {
        pa_status st = scratch_address(&scratch);
        if (st != PA_OK) return st;
    }
    return pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, dims,
                     max_context_len, partition_tokens, scratch, need > 0 ? kNoAllocScratchBytes : 0, stream);
}
