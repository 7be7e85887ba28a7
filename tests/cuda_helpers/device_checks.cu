// device_checks.cu -- test-only kernels exposing the product's device encoders (from the
// library's own device header) and cuRAND's independent Philox4_32_10 generator, so the GPU
// tests can compare them element by element with the CPU oracle.
#include <cuda_runtime.h>
#include <curand_kernel.h>

#include <cstdint>

#include "nvfp4_device.cuh"

using namespace nvfp4;

// x = bits start + i; out[i] = both nibbles of the packed RNE pair (x, x)
__global__ void k_e2m1_rne(uint32_t start, int64_t n, uint8_t* out) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float x = __uint_as_float(start + (uint32_t)i);
        out[i] = (uint8_t)e2m1x2_rne(x, x);
    }
}
// eight values per word, as the quantize kernels pack them: out[i] = codes of x[8i .. 8i + 7]
__global__ void k_e2m1x8(const float* x, int64_t nwords, uint32_t* out) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nwords; i += (int64_t)gridDim.x * blockDim.x) {
        const float* v = x + 8 * i;
        out[i] = e2m1x8_word(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
    }
}
__global__ void k_e2m1_sr_threshold(uint32_t start, int64_t n, uint32_t* out) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        out[i] = e2m1_sr_threshold((start + (uint32_t)i) & 0x7FFFFFFFu);
    }
}
__global__ void k_e2m1_sr(const float* x, const uint32_t* r, int64_t n, uint8_t* out) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        out[i] = (uint8_t)e2m1_sr(x[i], r[i]);
}
__global__ void k_e4m3(uint32_t start, int64_t n, uint8_t* out) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        out[i] = (uint8_t)e4m3_rne_sat(__uint_as_float(start + (uint32_t)i));
}
__global__ void k_e4m3_decode(float* out) {
    const int c = threadIdx.x;
    if (c < 127) out[c] = e4m3_decode((uint32_t)c);
}
__global__ void k_philox(uint64_t seed, uint32_t stream, uint64_t g0, int64_t n, uint32_t* out) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const U4 w = sr_words(seed, stream, g0 + (uint64_t)i);
        out[4 * i] = w.x;
        out[4 * i + 1] = w.y;
        out[4 * i + 2] = w.z;
        out[4 * i + 3] = w.w;
    }
}
// cuRAND: curand_init(seed, subsequence, offset) puts `subsequence` in the counter's upper
// 64 bits and offset/4 in the lower 64 bits; curand4 then returns that counter's block.
__global__ void k_curand_philox(uint64_t seed, uint32_t stream, uint64_t g0, int64_t n, uint32_t* out) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        curandStatePhilox4_32_10_t st;
        curand_init(seed, stream, 4ull * (g0 + (uint64_t)i), &st);
        const uint4 w = curand4(&st);
        out[4 * i] = w.x;
        out[4 * i + 1] = w.y;
        out[4 * i + 2] = w.z;
        out[4 * i + 3] = w.w;
    }
}
__global__ void k_rht16(const float* in, int64_t n, uint32_t signs, float* out) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = in[16 * i + j];
        rht16(v, signs);
#pragma unroll
        for (int j = 0; j < 16; ++j) out[16 * i + j] = v[j];
    }
}

static int grid(int64_t n) { int64_t g = (n + 255) / 256; return (int)(g < 4096 ? (g > 0 ? g : 1) : 4096); }

extern "C" {
int chk_e2m1_rne(uint32_t start, int64_t n, uint8_t* out) { k_e2m1_rne<<<grid(n), 256>>>(start, n, out); return (int)cudaDeviceSynchronize(); }
int chk_e2m1x8(const float* x, int64_t nwords, uint32_t* out) { k_e2m1x8<<<grid(nwords), 256>>>(x, nwords, out); return (int)cudaDeviceSynchronize(); }
int chk_e2m1_sr_threshold(uint32_t start, int64_t n, uint32_t* out) { k_e2m1_sr_threshold<<<grid(n), 256>>>(start, n, out); return (int)cudaDeviceSynchronize(); }
int chk_e2m1_sr(const float* x, const uint32_t* r, int64_t n, uint8_t* out) { k_e2m1_sr<<<grid(n), 256>>>(x, r, n, out); return (int)cudaDeviceSynchronize(); }
int chk_e4m3(uint32_t start, int64_t n, uint8_t* out) { k_e4m3<<<grid(n), 256>>>(start, n, out); return (int)cudaDeviceSynchronize(); }
int chk_e4m3_decode(float* out) { k_e4m3_decode<<<1, 128>>>(out); return (int)cudaDeviceSynchronize(); }
int chk_philox(uint64_t seed, uint32_t stream, uint64_t g0, int64_t n, uint32_t* out) { k_philox<<<grid(n), 256>>>(seed, stream, g0, n, out); return (int)cudaDeviceSynchronize(); }
int chk_curand_philox(uint64_t seed, uint32_t stream, uint64_t g0, int64_t n, uint32_t* out) { k_curand_philox<<<grid(n), 256>>>(seed, stream, g0, n, out); return (int)cudaDeviceSynchronize(); }
int chk_rht16(const float* in, int64_t n, uint32_t signs, float* out) { k_rht16<<<grid(n), 256>>>(in, n, signs, out); return (int)cudaDeviceSynchronize(); }
}
