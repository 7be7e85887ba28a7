// glue.cu -- GeLU forward/backward for the one-FFN training step (bf16 in/out, fp32 math).
// The pages do not describe the activation; the FFN step uses the exact (erf) form:
//   g  = h Phi(h),  Phi(h) = 0.5 erfc(-h / sqrt 2)  (= 0.5 (1 + erf(h / sqrt 2)) without the
//        cancellation of 1 + erf for negative h)
//   dh = dg * (Phi(h) + h * phi(h)),  phi = N(0,1) density.
// HBM-bound elementwise kernels: 16-byte loads and stores, grid-stride.
#include <cuda_runtime.h>

#include <cstdint>

#include "nvfp4_device.cuh"
#include "nvfp4_internal.h"

namespace nvfp4 {

__device__ __forceinline__ float gelu_f(float h) { return 0.5f * h * erfcf(h * -0.70710678118654752f); }

__device__ __forceinline__ float gelu_grad_f(float h) {
    const float cdf = 0.5f * erfcf(h * -0.70710678118654752f);
    const float pdf = 0.39894228040143268f * expf(-0.5f * h * h);
    return cdf + h * pdf;
}

__global__ void __launch_bounds__(256) gelu_fwd_kernel(const uint4* __restrict__ h, uint4* __restrict__ g, int64_t n8,
                                                       const uint16_t* __restrict__ h_tail, uint16_t* __restrict__ g_tail,
                                                       int tail) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        const uint4 v = h[i];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) o[j] = f32x2_to_bf16x2(gelu_f(bf16_lo(w[j])), gelu_f(bf16_hi(w[j])));
        g[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (blockIdx.x == 0 && (int)threadIdx.x < tail) {
        const float x = __uint_as_float((uint32_t)h_tail[threadIdx.x] << 16);
        g_tail[threadIdx.x] = (uint16_t)(f32x2_to_bf16x2(gelu_f(x), 0.0f) & 0xFFFFu);
    }
}

__global__ void __launch_bounds__(256) gelu_bwd_kernel(const uint4* __restrict__ h, const uint4* __restrict__ dg,
                                                       uint4* __restrict__ dh, int64_t n8,
                                                       const uint16_t* __restrict__ h_tail,
                                                       const uint16_t* __restrict__ dg_tail,
                                                       uint16_t* __restrict__ dh_tail, int tail) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        const uint4 v = h[i], d = dg[i];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        const uint32_t e[4] = {d.x, d.y, d.z, d.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            o[j] = f32x2_to_bf16x2(bf16_lo(e[j]) * gelu_grad_f(bf16_lo(w[j])), bf16_hi(e[j]) * gelu_grad_f(bf16_hi(w[j])));
        dh[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (blockIdx.x == 0 && (int)threadIdx.x < tail) {
        const float x = __uint_as_float((uint32_t)h_tail[threadIdx.x] << 16);
        const float y = __uint_as_float((uint32_t)dg_tail[threadIdx.x] << 16);
        dh_tail[threadIdx.x] = (uint16_t)(f32x2_to_bf16x2(y * gelu_grad_f(x), 0.0f) & 0xFFFFu);
    }
}

static int elementwise_grid(int64_t n8) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t want = (n8 + 255) / 256;
    int64_t cap = (int64_t)sms * 8;
    if (want < 1) want = 1;
    return (int)(want < cap ? want : cap);
}

cudaError_t launch_gelu_fwd(const uint16_t* h, uint16_t* g, int64_t n, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    const int64_t n8 = n / 8;
    const int tail = (int)(n - n8 * 8);
    gelu_fwd_kernel<<<elementwise_grid(n8), 256, 0, s>>>(reinterpret_cast<const uint4*>(h), reinterpret_cast<uint4*>(g),
                                                          n8, h + n8 * 8, g + n8 * 8, tail);
    return cudaGetLastError();
}

cudaError_t launch_gelu_bwd(const uint16_t* h, const uint16_t* dg, uint16_t* dh, int64_t n, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    const int64_t n8 = n / 8;
    const int tail = (int)(n - n8 * 8);
    gelu_bwd_kernel<<<elementwise_grid(n8), 256, 0, s>>>(reinterpret_cast<const uint4*>(h),
                                                          reinterpret_cast<const uint4*>(dg), reinterpret_cast<uint4*>(dh),
                                                          n8, h + n8 * 8, dg + n8 * 8, dh + n8 * 8, tail);
    return cudaGetLastError();
}

}  // namespace nvfp4
