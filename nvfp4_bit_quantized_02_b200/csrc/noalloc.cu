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
// by every call.  Device-side flags (non-finite input, a tile copy that ran out of its wait
// budget) stay set in the array until nvfp4_poll_noalloc reads and clears them; a flagged call's
// output is undefined.  The cached address belongs to the device's context at set-up time: it
// does not survive cudaDeviceReset of that device within the process.
#include <cuda_runtime.h>

#include <cstddef>
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

// Address of this device's scratch array (looked up once per device, with that device current).
nvfp4_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_LIMIT;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return NVFP4_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return NVFP4_OK;
}

}  // namespace

extern "C" nvfp4_status nvfp4_quantize_noalloc(const void* x, int64_t rows, int64_t cols, int64_t ldx, int along,
                                               nvfp4_round mode, nvfp4_block block, int rht, uint64_t rht_seed,
                                               uint64_t sr_seed, uint32_t stream_id, nvfp4_tensor* out,
                                               nvfp4_stream_t stream) {
    // the scratch this call needs must fit the fixed array
    if (nvfp4_workspace_bytes() > kNoAllocScratchBytes) return NVFP4_ERR_LIMIT;
    void* scratch = nullptr;
    if (nvfp4_status st = scratch_address(&scratch)) return st;
    return nvfp4_quantize(x, rows, cols, ldx, along, mode, block, rht, rht_seed, sr_seed, stream_id, out, scratch,
                          stream);
}

// The flags word of the scratch array, read and cleared after `stream` has finished: the same
// report as nvfp4_poll gives for a caller's workspace, without one.
extern "C" nvfp4_status nvfp4_poll_noalloc(nvfp4_stream_t stream) {
    void* scratch = nullptr;   // the set-up of this device (the address itself is not needed here)
    if (nvfp4_status st = scratch_address(&scratch)) return st;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    uint32_t flags = 0;
    if (cudaMemcpyFromSymbol(&flags, g_noalloc_scratch, sizeof(flags), offsetof(nvfp4::Workspace, flags),
                             cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    if (flags) {
        const uint32_t zero = 0;
        if (cudaMemcpyToSymbol(g_noalloc_scratch, &zero, sizeof(zero), offsetof(nvfp4::Workspace, flags),
                               cudaMemcpyHostToDevice) != cudaSuccess) {
            cudaGetLastError();
            return NVFP4_ERR_CUDA;
        }
    }
    if (flags & nvfp4::kFlagTimeout) return NVFP4_ERR_TIMEOUT;
    if (flags & nvfp4::kFlagNonFinite) return NVFP4_ERR_NONFINITE;
    return NVFP4_OK;
}
