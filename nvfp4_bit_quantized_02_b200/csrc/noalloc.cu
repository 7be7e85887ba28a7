// noalloc.cu -- nvfp4_quantize for callers that cannot hand the library a workspace.
//
// Some hosts own every byte of device memory themselves -- a framework whose caching
// allocator must be the only allocator, or a plugin interface that exposes no allocation
// hook -- so the code calling this library has no way to obtain the 256-byte workspace that
// nvfp4_quantize needs for its amax reduction.  This entry point runs the same quantization
// with the workspace placed in a fixed device array that belongs to the library itself.
//
// The array (kNoAllocScratchBytes bytes) lives in this file; every GPU that loads the library
// keeps it until the process exits.  Host code cannot use the array's name as a device
// address, so the first call on each device looks the address up with cudaGetSymbolAddress
// (with that device current) and caches it; make that first call before any stream capture.
// All calls share the one array: calls whose work overlaps on the GPU (other streams, other
// host threads) race on it and must be serialised by the caller.  The amax slots are cleared
// by every call; device-side flags (non-finite input) are not reported by this variant.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "nvfp4.h"
#include "nvfp4_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 256;   // room for exactly one workspace
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_addr[kMaxDevices];

}  // namespace

extern "C" nvfp4_status nvfp4_quantize_noalloc(const void* x, int64_t rows, int64_t cols, int64_t ldx, int along,
                                               nvfp4_round mode, nvfp4_block block, int rht, uint64_t rht_seed,
                                               uint64_t sr_seed, uint32_t stream_id, nvfp4_tensor* out,
                                               nvfp4_stream_t stream) {
    // the scratch this call needs must fit the fixed array
    if (nvfp4_workspace_bytes() > kNoAllocScratchBytes) return NVFP4_ERR_LIMIT;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_LIMIT;
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_setup_mu);
        if (!g_scratch_addr[dev]) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
                cudaGetLastError();
                return NVFP4_ERR_CUDA;
            }
            g_scratch_addr[dev] = p;
        }
        scratch = g_scratch_addr[dev];
    }
    return nvfp4_quantize(x, rows, cols, ldx, along, mode, block, rht, rht_seed, sr_seed, stream_id, out, scratch,
                          stream);
}
