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

// ---------------------------------------------------------------------------------------
// GeLU forward or backward with the amax of its bf16 output fused in (the amax pass of the
// next quantize, which reads this output, is then skipped): a thread takes a 16-row x 4-column
// patch of the [rows][cols] output, writes it, and reduces its plain magnitudes (as packed
// bf16 integers) and its 16-point RHT along rows (fp32), exactly as the amax pass does.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint2 ld_patch_row(const uint16_t* p) { return *reinterpret_cast<const uint2*>(p); }

__device__ __forceinline__ uint32_t warp_max_u32_g(uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

__device__ __forceinline__ void block_max_to(uint32_t v, uint32_t* dst, uint32_t* red) {
    v = warp_max_u32_g(v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < (int)(blockDim.x >> 5) ? red[lane] : 0u;
        v = warp_max_u32_g(v);
        if (lane == 0 && v) atomicMax(dst, v);
    }
    __syncthreads();
}

template <bool BWD>
__global__ void __launch_bounds__(256, 2) gelu_amax_kernel(const uint16_t* __restrict__ h, const uint16_t* __restrict__ dg,
                                                        uint16_t* __restrict__ out, int64_t rows, int64_t cols,
                                                        uint32_t signs, uint32_t* __restrict__ amax_plain,
                                                        uint32_t* __restrict__ amax_rht, uint32_t* __restrict__ flags) {
    __shared__ uint32_t red[8];
    const int64_t cpr = cols >> 2;
    const int64_t total = (rows >> 4) * cpr;
    uint32_t m = 0;
    float mr = 0.0f;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < total; u += (int64_t)gridDim.x * blockDim.x) {
        const int64_t g = u / cpr, k = u - g * cpr;
        const int64_t base = (g << 4) * cols + (k << 2);
        uint2 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint2 x = ld_patch_row(h + base + i * cols);
            if (BWD) {
                const uint2 d = ld_patch_row(dg + base + i * cols);
                v[i].x = f32x2_to_bf16x2(bf16_lo(d.x) * gelu_grad_f(bf16_lo(x.x)), bf16_hi(d.x) * gelu_grad_f(bf16_hi(x.x)));
                v[i].y = f32x2_to_bf16x2(bf16_lo(d.y) * gelu_grad_f(bf16_lo(x.y)), bf16_hi(d.y) * gelu_grad_f(bf16_hi(x.y)));
            } else {
                v[i].x = f32x2_to_bf16x2(gelu_f(bf16_lo(x.x)), gelu_f(bf16_hi(x.x)));
                v[i].y = f32x2_to_bf16x2(gelu_f(bf16_lo(x.y)), gelu_f(bf16_hi(x.y)));
            }
            *reinterpret_cast<uint2*>(out + base + i * cols) = v[i];
            m = __vmaxu2(m, v[i].x & 0x7FFF7FFFu);
            m = __vmaxu2(m, v[i].y & 0x7FFF7FFFu);
        }
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            float a[16], b[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t w = p == 0 ? v[i].x : v[i].y;
                a[i] = bf16_lo(w);
                b[i] = bf16_hi(w);
            }
            rht16(a, signs);
            rht16(b, signs);
#pragma unroll
            for (int i = 0; i < 16; ++i) mr = fmaxf(mr, fmaxf(fabsf(a[i]), fabsf(b[i])));
        }
    }
    const uint32_t mag = max(m & 0xFFFFu, m >> 16);
    if (mag >= 0x7F80u || !(mr < __int_as_float(0x7F800000))) atomicOr(flags, kFlagNonFinite);
    block_max_to(mag << 16, amax_plain, red);
    block_max_to(__float_as_uint(mr), amax_rht, red);
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

cudaError_t launch_gelu_amax(bool bwd, const uint16_t* h, const uint16_t* dg, uint16_t* out, int64_t rows,
                             int64_t cols, uint32_t signs, uint32_t* amax_plain, uint32_t* amax_rht, uint32_t* flags,
                             cudaStream_t s) {
    const int64_t units = (rows >> 4) * (cols >> 2);
    if (units == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (units + 255) / 256, cap = (int64_t)sms * 4;
    const int grid = (int)(want < cap ? want : cap);
    if (bwd)
        gelu_amax_kernel<true><<<grid, 256, 0, s>>>(h, dg, out, rows, cols, signs, amax_plain, amax_rht, flags);
    else
        gelu_amax_kernel<false><<<grid, 256, 0, s>>>(h, nullptr, out, rows, cols, signs, amax_plain, amax_rht, flags);
    return cudaGetLastError();
}

}  // namespace nvfp4
