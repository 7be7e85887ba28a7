// glue.cu -- GeLU forward/backward for the one-FFN training step (bf16 in/out, fp32 math), and
// the bf16 transpose of the BF16 path.
// The pages do not describe the activation; the FFN step uses the exact (erf) form:
//   g  = h Phi(h),  Phi the standard normal distribution function,
//   dh = dg * (Phi(h) + h * phi(h)),  phi = N(0,1) density.
// Phi comes from erfc(|h| / sqrt 2) through the Chebyshev fit of erfc(z) exp(z^2) in
// t = 1 / (1 + z/2) published by Press, Teukolsky, Vetterling and Flannery (Numerical Recipes,
// 2nd ed., section 6.2), whose fractional error is below 1.2e-7 for every z >= 0.
// Two evaluations:
//   - pairs (|h| <= 12, the bulk): two elements per f32x2 instruction, t from the approximate
//     reciprocal and e^x as 2^(x log2 e) on the multi-function unit.  The fp32 rounding of the
//     exponent's argument (|x| up to ~75 at |h| = 12) dominates the error: relative ~1e-5 at the
//     far end, ~1e-6 for |h| < 3, against the bf16 results' half-step of 2^-9;
//   - scalar (|h| > 12, inf, NaN): IEEE reciprocal and expf, with the far tail scaled (below).
// The tests sweep every finite bf16 input against the fp64 oracle (within one bf16 step, more
// than 99.9 % exact).  The library erfcf took about three times the instructions and made these
// kernels compute-bound; the pair form streams at about the speed of a copy.
// Elementwise kernels: 16-byte loads and stores, grid-stride.
#include <cuda_runtime.h>

#include <cstdint>

#include "nvfp4_device.cuh"
#include "nvfp4_internal.h"

namespace nvfp4 {

// erfc(z) for z >= 0, times e^lnscale (the scale lets a caller keep the far tail, where erfc
// falls below the normal fp32 range, at full precision)
__device__ __forceinline__ float erfc_pos(float z, float lnscale) {
    const float t = __frcp_rn(fmaf(0.5f, z, 1.0f));
    float p = 0.17087277f;
    p = fmaf(t, p, -0.82215223f);
    p = fmaf(t, p, 1.48851587f);
    p = fmaf(t, p, -1.13520398f);
    p = fmaf(t, p, 0.27886807f);
    p = fmaf(t, p, -0.18628806f);
    p = fmaf(t, p, 0.09678418f);
    p = fmaf(t, p, 0.37409196f);
    p = fmaf(t, p, 1.00002368f);
    return t * expf(fmaf(-z, z, fmaf(t, p, -1.26551223f)) + lnscale);
}

// Phi(h), the standard normal distribution function
__device__ __forceinline__ float normal_cdf(float h) {
    const float e = erfc_pos(fabsf(h) * 0.70710678118654752f, 0.0f);
    return h >= 0.0f ? fmaf(-0.5f, e, 1.0f) : 0.5f * e;
}

__device__ __forceinline__ float gelu_f(float h) { return h * normal_cdf(h); }

__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ float ex2_approx(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}
// e^x for a pair, x >= -80 (normal results)
__device__ __forceinline__ uint64_t exp_pair(uint64_t x) {
    float a, b;
    f2_split(f2_mul(x, f2c(1.4426950408889634f)), a, b);
    return f2(ex2_approx(a), ex2_approx(b));
}
// erfc(|h| / sqrt 2) of a pair with |h| <= 12, and m2 = -h^2 / 2 (exact: h is a bf16 value)
__device__ __forceinline__ uint64_t erfc_pair(float hl, float hh, uint64_t& m2) {
    const float dl = fmaf(fabsf(hl), 0.35355339059327376f, 1.0f), dh = fmaf(fabsf(hh), 0.35355339059327376f, 1.0f);
    const uint64_t t = f2(rcp_approx(dl), rcp_approx(dh));   // 1 / (1 + z/2)
    uint64_t p = f2c(0.17087277f);
    p = f2_fma(t, p, f2c(-0.82215223f));
    p = f2_fma(t, p, f2c(1.48851587f));
    p = f2_fma(t, p, f2c(-1.13520398f));
    p = f2_fma(t, p, f2c(0.27886807f));
    p = f2_fma(t, p, f2c(-0.18628806f));
    p = f2_fma(t, p, f2c(0.09678418f));
    p = f2_fma(t, p, f2c(0.37409196f));
    p = f2_fma(t, p, f2c(1.00002368f));
    const uint64_t h2 = f2(hl, hh);
    m2 = f2_mul(f2_mul(h2, f2c(-0.5f)), h2);
    return f2_mul(t, exp_pair(f2_add(f2_fma(t, p, f2c(-1.26551223f)), m2)));
}
// GeLU of a bf16 pair (|h| <= 12): h Phi(h) = max(h, 0) - |h| erfc(|h| / sqrt 2) / 2
__device__ __forceinline__ uint32_t gelu_pair(uint32_t w) {
    const float hl = bf16_lo(w), hh = bf16_hi(w);
    uint64_t m2;
    const uint64_t e = erfc_pair(hl, hh, m2);
    float gl, gh;
    f2_split(f2_fma(f2(fabsf(hl) * -0.5f, fabsf(hh) * -0.5f), e, f2(fmaxf(hl, 0.0f), fmaxf(hh, 0.0f))), gl, gh);
    return f32x2_to_bf16x2(gl, gh);
}
// dg GeLU'(h) of a bf16 pair (|h| <= 12): Phi(h) = [h >= 0] -+ erfc / 2, phi(h) = e^(-h^2/2) / sqrt(2 pi)
__device__ __forceinline__ uint32_t gelu_bwd_pair(uint32_t w, uint32_t d) {
    const float hl = bf16_lo(w), hh = bf16_hi(w);
    uint64_t m2;
    const uint64_t e = erfc_pair(hl, hh, m2);
    const uint64_t cdf = f2_fma(f2(hl >= 0.0f ? -0.5f : 0.5f, hh >= 0.0f ? -0.5f : 0.5f), e,
                                f2(hl >= 0.0f ? 1.0f : 0.0f, hh >= 0.0f ? 1.0f : 0.0f));
    const uint64_t hc = f2_mul(f2(hl, hh), f2c(0.39894228040143268f));
    float rl, rh;
    f2_split(f2_mul(f2_fma(hc, exp_pair(m2), cdf), bf16x2_to_f2(d)), rl, rh);
    return f32x2_to_bf16x2(rl, rh);
}
// a bf16 pair whose magnitudes are both <= 12 (neither inf nor NaN)
__device__ __forceinline__ bool pair_in_range(uint32_t w) {
    return __vcmpleu2(w & 0x7FFF7FFFu, 0x41404140u) == 0xFFFFFFFFu;
}
__device__ __forceinline__ bool quad_in_range(const uint4& v) {
    const uint32_t m = __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu), __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
    return max(m & 0xFFFFu, m >> 16) <= 0x4140u;
}
__device__ __forceinline__ uint32_t gelu_word(uint32_t w) {
    return pair_in_range(w) ? gelu_pair(w) : f32x2_to_bf16x2(gelu_f(bf16_lo(w)), gelu_f(bf16_hi(w)));
}

// dg * GeLU'(h) = dg * (Phi(h) + h phi(h)).  Below h = -12 both terms fall towards the subnormal
// fp32 range, where they would keep only a few significant bits that a large dg could lift back
// into bf16's normal range: there they are evaluated scaled by 2^64 (inside the exponentials) and
// the scale is undone after the product with dg.
__device__ __forceinline__ float gelu_bwd_f(float h, float dg) {
    const bool tail = h < -12.0f;
    const float lnscale = tail ? 44.361419555836500f : 0.0f;   // 64 ln 2
    const float z = fabsf(h) * 0.70710678118654752f;
    const float e = erfc_pos(z, lnscale);
    const float cdf = h >= 0.0f ? fmaf(-0.5f, e, 1.0f) : 0.5f * e;
    const float pdf = 0.39894228040143268f * expf(fmaf(-0.5f * h, h, lnscale));
    const float r = dg * fmaf(h, pdf, cdf);
    return tail ? r * 5.42101086242752217e-20f : r;                // 2^-64
}

__device__ __forceinline__ uint32_t gelu_bwd_word(uint32_t w, uint32_t d) {
    return pair_in_range(w) ? gelu_bwd_pair(w, d)
                            : f32x2_to_bf16x2(gelu_bwd_f(bf16_lo(w), bf16_lo(d)), gelu_bwd_f(bf16_hi(w), bf16_hi(d)));
}

__global__ void __launch_bounds__(256) gelu_fwd_kernel(const uint4* __restrict__ h, uint4* __restrict__ g, int64_t n8,
                                                       const uint16_t* __restrict__ h_tail, uint16_t* __restrict__ g_tail,
                                                       int tail) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        const uint4 v = h[i];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
        if (quad_in_range(v)) {
#pragma unroll
            for (int j = 0; j < 4; ++j) o[j] = gelu_pair(w[j]);
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) o[j] = gelu_word(w[j]);
        }
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
        if (quad_in_range(v)) {
#pragma unroll
            for (int j = 0; j < 4; ++j) o[j] = gelu_bwd_pair(w[j], e[j]);
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) o[j] = gelu_bwd_word(w[j], e[j]);
        }
        dh[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (blockIdx.x == 0 && (int)threadIdx.x < tail) {
        const float x = __uint_as_float((uint32_t)h_tail[threadIdx.x] << 16);
        const float y = __uint_as_float((uint32_t)dg_tail[threadIdx.x] << 16);
        dh_tail[threadIdx.x] = (uint16_t)(f32x2_to_bf16x2(gelu_bwd_f(x, y), 0.0f) & 0xFFFFu);
    }
}

// ---------------------------------------------------------------------------------------
// GeLU forward or backward with the amax of its bf16 output fused in (the amax pass of the
// next quantize, which reads this output, is then skipped).  A CTA walks 32-row x 256-column
// tiles of the [rows][cols] output:
//   1. each thread streams four 16-byte chunks of the tile (the plain kernel's access pattern),
//      stores their GeLU to global memory and to a shared-memory copy of the tile, and keeps the
//      packed-integer max of the bf16 magnitudes;
//   2. after a barrier each thread takes one column pair of one 16-row group from shared memory
//      (a warp reads 32 consecutive words of a row: no bank conflicts) and applies the 16-point
//      RHT along the rows to it (f32x2 pairs), keeping the max magnitude -- exactly what the amax
//      pass computes from this output.
// ---------------------------------------------------------------------------------------
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

constexpr int kGaRows = 32, kGaWords = 128;   // a tile: 32 rows x 256 bf16 (128 words a row)

template <bool BWD>
__global__ void __launch_bounds__(256) gelu_amax_kernel(const uint16_t* __restrict__ h, const uint16_t* __restrict__ dg,
                                                        uint16_t* __restrict__ out, int64_t rows, int64_t cols,
                                                        const SignMasks sm, uint32_t* __restrict__ amax_plain,
                                                        uint32_t* __restrict__ amax_rht, uint32_t* __restrict__ flags) {
    __shared__ __align__(16) uint32_t tile[kGaRows][kGaWords];
    __shared__ uint32_t red[8];
    const int tid = threadIdx.x;
    const int64_t ntr = (rows + kGaRows - 1) / kGaRows, ntc = (cols + 2 * kGaWords - 1) / (2 * kGaWords);
    const int64_t ntiles = ntr * ntc;
    uint32_t m = 0;
    float mr = 0.0f;
    for (int64_t it = blockIdx.x; it < ntiles; it += gridDim.x) {
        const int64_t r0 = (it / ntc) * kGaRows, c0 = (it % ntc) * (2 * kGaWords);
        // 1. GeLU of the tile: chunk j = 8 bf16 at row j / 32, columns 8 (j % 32) ..
        uint4 v[4], d[4];
        bool ok[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = tid + 256 * u, r = j >> 5, q = j & 31;
            ok[u] = r0 + r < rows && c0 + 8 * q < cols;
            const int64_t off = (r0 + r) * cols + c0 + 8 * q;
            v[u] = ok[u] ? *reinterpret_cast<const uint4*>(h + off) : make_uint4(0, 0, 0, 0);
            if (BWD) d[u] = ok[u] ? *reinterpret_cast<const uint4*>(dg + off) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = tid + 256 * u, r = j >> 5, q = j & 31;
            const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
            uint32_t o[4];
            if (BWD) {
                const uint32_t e[4] = {d[u].x, d[u].y, d[u].z, d[u].w};
                if (quad_in_range(v[u])) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) o[k] = gelu_bwd_pair(w[k], e[k]);
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k) o[k] = gelu_bwd_word(w[k], e[k]);
                }
            } else {
                if (quad_in_range(v[u])) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) o[k] = gelu_pair(w[k]);
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k) o[k] = gelu_word(w[k]);
                }
            }
            const uint4 ov = ok[u] ? make_uint4(o[0], o[1], o[2], o[3]) : make_uint4(0, 0, 0, 0);
            if (ok[u]) *reinterpret_cast<uint4*>(out + (r0 + r) * cols + c0 + 8 * q) = ov;
            *reinterpret_cast<uint4*>(&tile[r][4 * q]) = ov;
            m = __vmaxu2(m, __vmaxu2(__vmaxu2(ov.x & 0x7FFF7FFFu, ov.y & 0x7FFF7FFFu),
                                     __vmaxu2(ov.z & 0x7FFF7FFFu, ov.w & 0x7FFF7FFFu)));
        }
        __syncthreads();
        // 2. the RHT amax of column pair c of 16-row group g
        {
            const int g = tid >> 7, c = tid & (kGaWords - 1);
            if (r0 + 16 * g < rows && c0 + 2 * c < cols) {
                uint64_t f[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) f[i] = bf16x2_to_f2(tile[16 * g + i][c] ^ sm.m[i]);
                rht16_pairs(f);
#pragma unroll
                for (int i = 0; i < 16; i += 2) {
                    float a0, a1, b0, b1;
                    f2_split(f[i], a0, a1);
                    f2_split(f[i + 1], b0, b1);
                    mr = max3_abs(max3_abs(mr, a0, a1), b0, b1);
                }
            }
        }
        __syncthreads();   // the tile copy is free for the next tile
    }
    const uint32_t mag = max(m & 0xFFFFu, m >> 16);
    if (mag >= 0x7F80u || !(mr < __int_as_float(0x7F800000))) atomicOr(flags, kFlagNonFinite);
    block_max_to(mag << 16, amax_plain, red);
    block_max_to(__float_as_uint(mr), amax_rht, red);
}

// ---------------------------------------------------------------------------------------
// bf16 transpose xt[c][r] = x[r][c] (the K-major operands of the BF16 path's dgrad and wgrad):
// 64 x 64 tiles through shared memory, 16-byte loads and stores on both sides; rows % 8 == 0,
// cols % 8 == 0.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) transpose_bf16_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t cols,
                                                             int64_t ldx, uint16_t* __restrict__ xt, int64_t ldt) {
    __shared__ uint16_t t[64][64 + 2];
    const int tid = threadIdx.x;
    const int64_t ntc = (cols + 63) / 64, ntiles = ((rows + 63) / 64) * ntc;
    for (int64_t it = blockIdx.x; it < ntiles; it += gridDim.x) {
        const int64_t r0 = (it / ntc) * 64, c0 = (it % ntc) * 64;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int j = tid + 256 * u, r = j >> 3, ch = j & 7;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (r0 + r < rows && c0 + ch * 8 < cols) v = *reinterpret_cast<const uint4*>(x + (r0 + r) * ldx + c0 + ch * 8);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                t[r][ch * 8 + 2 * e] = (uint16_t)(w[e] & 0xFFFFu);
                t[r][ch * 8 + 2 * e + 1] = (uint16_t)(w[e] >> 16);
            }
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int j = tid + 256 * u, c = j >> 3, ch = j & 7;
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                w[e] = (uint32_t)t[ch * 8 + 2 * e][c] | ((uint32_t)t[ch * 8 + 2 * e + 1][c] << 16);
            if (c0 + c < cols && r0 + ch * 8 < rows)
                *reinterpret_cast<uint4*>(xt + (c0 + c) * ldt + r0 + ch * 8) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        __syncthreads();
    }
}

cudaError_t launch_transpose_bf16(const uint16_t* x, int64_t rows, int64_t cols, int64_t ldx, uint16_t* xt, int64_t ldt,
                                  cudaStream_t s) {
    const int64_t tiles = ((rows + 63) / 64) * ((cols + 63) / 64);
    if (tiles == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t cap = (int64_t)sms * 8;
    transpose_bf16_kernel<<<(int)(tiles < cap ? tiles : cap), 256, 0, s>>>(x, rows, cols, ldx, xt, ldt);
    return cudaGetLastError();
}

static int elementwise_grid(int64_t n8) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t want = (n8 + 255) / 256;
    int64_t cap = (int64_t)sms * 16;
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
    const int64_t tiles = ((rows + kGaRows - 1) / kGaRows) * ((cols + 2 * kGaWords - 1) / (2 * kGaWords));
    if (rows == 0 || cols == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t cap = (int64_t)sms * 8;   // resident CTAs: 16.5 KiB of shared memory each
    const int grid = (int)(tiles < cap ? tiles : cap);
    if (bwd)
        gelu_amax_kernel<true><<<grid, 256, 0, s>>>(h, dg, out, rows, cols, sign_masks(signs), amax_plain, amax_rht, flags);
    else
        gelu_amax_kernel<false><<<grid, 256, 0, s>>>(h, nullptr, out, rows, cols, sign_masks(signs), amax_plain,
                                                     amax_rht, flags);
    return cudaGetLastError();
}

}  // namespace nvfp4
