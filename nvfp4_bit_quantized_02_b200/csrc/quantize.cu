// quantize.cu -- NVFP4 quantization kernels for sm_100a.
//
// gist.science "Pretraining Large Language Models with NVFP4", Technische Zusammenfassung:
//   2.A    E2M1 elements, one E4M3 scale per 16 elements, one fp32 tensor scale from amax;
//   2.B.2  16-point Random Hadamard Transform on the Wgrad inputs (along tokens);
//   2.B.3  16x16 weight blocks, the same quantized weight forward and backward (transposed);
//   2.B.4  stochastic rounding for gradients, round-to-nearest-even elsewhere.
//
// Two passes over the bf16 input (the tensor scale needs the amax of the whole tensor):
//   1. amax: 16-byte loads, bf16 magnitudes reduced as packed 16-bit integers (the bf16
//      magnitude order is the integer order of its low 15 bits), RHT outputs reduced in
//      fp32; one atomicMax per CTA on the fp32 bit pattern (non-negative floats order like
//      unsigned ints, and max does not depend on the order of the reduction).
//   2. quantize: a thread owns a 16-row x 8-column patch (16 x 16-byte loads).  From the same
//      registers it can emit
//        - the ROW form (K = columns): a 1x16 block is a lane pair, one shuffle for its amax;
//          each lane writes 4 code bytes per row (a warp writes 128 contiguous bytes);
//        - the COL form (K = rows, the transposed wgrad/dgrad operand): a 1x16 block is one
//          column of the patch, optionally rotated by the 16-point butterfly; codes and
//          scales are staged in shared memory and written as contiguous row segments.
//      16x16 tiles (weights) are a lane pair's 16x16 patch; both forms share its scale.
// The quantize pass walks the tiles in reverse order of the amax pass so its first wave
// reads what the amax pass left in L2.
#include <cuda_runtime.h>

#include <cstdint>

#include "nvfp4_device.cuh"
#include "nvfp4_internal.h"

namespace nvfp4 {

// ---------------------------------------------------------------------------------------
// loads
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t mag_max2(uint32_t m, uint32_t pair) {
    return __vmaxu2(m, pair & 0x7FFF7FFFu);
}

__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// Reduce per-thread maxima (fp32 bit patterns of non-negative values) to one atomicMax.
__device__ __forceinline__ void block_atomic_max(uint32_t v, uint32_t* dst, uint32_t* red) {
    v = warp_max_u32(v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < (int)(blockDim.x >> 5) ? red[lane] : 0u;
        v = warp_max_u32(v);
        if (lane == 0 && v) atomicMax(dst, v);
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------------------
// pass 1a: plain amax over a [rows][cols] bf16 tensor with leading dimension ld
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) amax_plain_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                         int64_t cols, int64_t ld,
                                                         uint32_t* __restrict__ amax_bits,
                                                         uint32_t* __restrict__ flags) {
    __shared__ uint32_t red[8];
    const int64_t cpr = cols >> 3;  // 16-byte chunks per row
    const int64_t total = rows * cpr;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    uint32_t m = 0;
    int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    // four independent loads in flight per iteration
    for (; c + 3 * stride < total; c += 4 * stride) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t cc = c + u * stride;
            const int64_t r = cc / cpr, k = cc - r * cpr;
            v[u] = ldg_stream(x + r * ld + (k << 3));
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            m = mag_max2(m, v[u].x);
            m = mag_max2(m, v[u].y);
            m = mag_max2(m, v[u].z);
            m = mag_max2(m, v[u].w);
        }
    }
    for (; c < total; c += stride) {
        const int64_t r = c / cpr, k = c - r * cpr;
        const uint4 v = ldg_stream(x + r * ld + (k << 3));
        m = mag_max2(m, v.x);
        m = mag_max2(m, v.y);
        m = mag_max2(m, v.z);
        m = mag_max2(m, v.w);
    }
    uint32_t mag = max(m & 0xFFFFu, m >> 16);
    if (mag >= 0x7F80u) atomicOr(flags, kFlagNonFinite);  // Inf (0x7F80) or NaN
    block_atomic_max(mag << 16, amax_bits, red);
}

// ---------------------------------------------------------------------------------------
// pass 1b: plain amax and amax of the 16-point RHT along rows (one read).  A thread takes a
// 16-row x 8-column patch; rows % 16 == 0, cols % 8 == 0.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) amax_rht_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                       int64_t cols, int64_t ld, uint32_t signs,
                                                       uint32_t* __restrict__ amax_plain_bits,
                                                       uint32_t* __restrict__ amax_rht_bits,
                                                       uint32_t* __restrict__ flags) {
    __shared__ uint32_t red[8];
    const int64_t cpr = cols >> 3;
    const int64_t groups = rows >> 4;
    const int64_t total = groups * cpr;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    uint32_t m = 0;
    float mr = 0.0f;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < total; u += stride) {
        const int64_t g = u / cpr, k = u - g * cpr;
        const uint16_t* base = x + (g << 4) * ld + (k << 3);
        uint4 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = ldg_stream(base + i * ld);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            m = mag_max2(m, v[i].x);
            m = mag_max2(m, v[i].y);
            m = mag_max2(m, v[i].z);
            m = mag_max2(m, v[i].w);
        }
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            float a[16], b[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t w = p == 0 ? v[i].x : p == 1 ? v[i].y : p == 2 ? v[i].z : v[i].w;
                a[i] = bf16_lo(w);
                b[i] = bf16_hi(w);
            }
            rht16(a, signs);
            rht16(b, signs);
#pragma unroll
            for (int i = 0; i < 16; ++i) mr = fmaxf(mr, fmaxf(fabsf(a[i]), fabsf(b[i])));
        }
    }
    uint32_t mag = max(m & 0xFFFFu, m >> 16);
    if (mag >= 0x7F80u || !(mr < __int_as_float(0x7F800000))) atomicOr(flags, kFlagNonFinite);
    block_atomic_max(mag << 16, amax_plain_bits, red);
    block_atomic_max(__float_as_uint(mr), amax_rht_bits, red);
}

// ---------------------------------------------------------------------------------------
// pass 2: the tile quantizer
// ---------------------------------------------------------------------------------------
constexpr int kTileRows = 64;    // 4 warps x 16 rows
constexpr int kTileCols = 256;   // 32 lanes x 8 columns
constexpr int kQuantThreads = 128;

__device__ __forceinline__ uint32_t word_of(const uint4& v, int p) {
    return p == 0 ? v.x : p == 1 ? v.y : p == 2 ? v.z : v.w;
}

// Encode 8 fp32 values (already multiplied by r_b) with RNE into 8 nibbles, element 0 lowest.
__device__ __forceinline__ uint32_t encode8_rne(const float (&u)[8]) {
    return e2m1x2_rne(u[0], u[1]) | (e2m1x2_rne(u[2], u[3]) << 8) | (e2m1x2_rne(u[4], u[5]) << 16) |
           (e2m1x2_rne(u[6], u[7]) << 24);
}

template <bool ROW, bool COL>
__global__ void __launch_bounds__(kQuantThreads) quantize_tile_kernel(QuantParams p) {
    // COL staging: codes [256 columns][4 row groups x 8 bytes], scales [256][4]
    __shared__ __align__(16) uint8_t s_codes[COL ? kTileCols * 32 : 16];
    __shared__ __align__(16) uint8_t s_scales[COL ? kTileCols * 4 : 16];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t rows = p.rows, cols = p.cols, ld = p.ld;
    const int64_t ntr = (rows + kTileRows - 1) / kTileRows;
    const int64_t ntc = (cols + kTileCols - 1) / kTileCols;
    const int64_t ntiles = ntr * ntc;

    const float amax_r = __uint_as_float(ROW ? *p.amax_row : 0u);
    const float amax_c = __uint_as_float(COL ? *p.amax_col : 0u);
    const float senc_r = encode_scale(amax_r);
    const float senc_c = encode_scale(amax_c);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        if (ROW) *p.st_row = decode_scale(amax_r);
        if (COL) *p.st_col = decode_scale(amax_c);
    }

    for (int64_t it = blockIdx.x; it < ntiles; it += gridDim.x) {
        const int64_t t = ntiles - 1 - it;  // reverse of the amax pass
        const int64_t tr = t / ntc, tc = t - tr * ntc;
        const int64_t r0 = tr * kTileRows + warp * 16;
        const int64_t c0 = tc * kTileCols + lane * 8;
        const bool col_ok = c0 < cols;
        const bool grp_ok = r0 < rows;

        uint4 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            v[i] = make_uint4(0u, 0u, 0u, 0u);
            if (col_ok && r0 + i < rows) v[i] = ldg_stream(p.x + (r0 + i) * ld + c0);
        }

        // ---- 16x16 tile scale (weights): max over the lane pair's 16x16 patch --------------
        BlockScale tile_sc{0u, 0.0f};
        if (p.block16) {
            uint32_t m = 0;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                m = mag_max2(m, v[i].x);
                m = mag_max2(m, v[i].y);
                m = mag_max2(m, v[i].z);
                m = mag_max2(m, v[i].w);
            }
            m = max(m & 0xFFFFu, m >> 16);
            m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
            // the tile amax is a bf16 magnitude; both forms see the same tensor amax
            tile_sc = block_scale(__uint_as_float(m << 16), ROW ? senc_r : senc_c);
            if (col_ok && grp_ok && (lane & 1) == 0) {
                if (ROW && p.tiles_row) p.tiles_row[(r0 >> 4) * (cols >> 4) + (c0 >> 4)] = (uint8_t)tile_sc.code;
                if (COL && p.tiles_col) p.tiles_col[(c0 >> 4) * (rows >> 4) + (r0 >> 4)] = (uint8_t)tile_sc.code;
            }
        }

        // ---- ROW form: K = columns ------------------------------------------------------------
        if (ROW) {
            const int64_t kb = c0 >> 4;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int64_t r = r0 + i;
                float x8[8];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t w = word_of(v[i], q);
                    x8[2 * q] = bf16_lo(w);
                    x8[2 * q + 1] = bf16_hi(w);
                }
                BlockScale sc = tile_sc;
                if (!p.block16) {
                    uint32_t m = 0;
#pragma unroll
                    for (int q = 0; q < 4; ++q) m = mag_max2(m, word_of(v[i], q));
                    m = max(m & 0xFFFFu, m >> 16);
                    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
                    sc = block_scale(__uint_as_float(m << 16), senc_r);
                }
                float u[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) u[e] = __fmul_rn(x8[e], sc.mult);
                uint32_t packed;
                if (p.sr_row) {
                    const uint64_t g = ((uint64_t)r * (uint64_t)cols + (uint64_t)c0) >> 3;
                    const U4 w = sr_words(p.sr_seed, p.stream_row, g);
                    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
                    packed = 0;
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        packed |= e2m1_sr(u[e], (ws[e >> 1] >> (16 * (e & 1))) & 0xFFFFu) << (4 * e);
                } else {
                    packed = encode8_rne(u);
                }
                if (col_ok && r < rows) {
                    *reinterpret_cast<uint32_t*>(p.codes_row + r * (cols >> 1) + (c0 >> 1)) = packed;
                    if ((lane & 1) == 0) p.scales_row[scale_offset(r, kb, p.nkt_row)] = (uint8_t)sc.code;
                }
            }
        }

        // ---- COL form: K = rows (transposed operand), optional RHT -------------------------
        if (COL) {
            U4 rw[16];
            if (p.sr_col) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint64_t g = ((uint64_t)(r0 + i) * (uint64_t)cols + (uint64_t)c0) >> 3;
                    rw[i] = sr_words(p.sr_seed, p.stream_col, g);
                }
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float a[16], b[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint32_t w = word_of(v[i], q);
                    a[i] = bf16_lo(w);
                    b[i] = bf16_hi(w);
                }
                if (p.rht_col) {
                    rht16(a, p.signs);
                    rht16(b, p.signs);
                }
                BlockScale sa = tile_sc, sb = tile_sc;
                if (!p.block16) {
                    float ma = 0.0f, mb = 0.0f;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        ma = fmaxf(ma, fabsf(a[i]));
                        mb = fmaxf(mb, fabsf(b[i]));
                    }
                    sa = block_scale(ma, senc_c);
                    sb = block_scale(mb, senc_c);
                }
                uint32_t ca0 = 0, ca1 = 0, cb0 = 0, cb1 = 0;
                if (p.sr_col) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const uint32_t w = q == 0 ? rw[i].x : q == 1 ? rw[i].y : q == 2 ? rw[i].z : rw[i].w;
                        const uint32_t na = e2m1_sr(__fmul_rn(a[i], sa.mult), w & 0xFFFFu);
                        const uint32_t nb = e2m1_sr(__fmul_rn(b[i], sb.mult), w >> 16);
                        if (i < 8) {
                            ca0 |= na << (4 * i);
                            cb0 |= nb << (4 * i);
                        } else {
                            ca1 |= na << (4 * (i - 8));
                            cb1 |= nb << (4 * (i - 8));
                        }
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        ca0 |= e2m1x2_rne(__fmul_rn(a[2 * j], sa.mult), __fmul_rn(a[2 * j + 1], sa.mult)) << (8 * j);
                        ca1 |= e2m1x2_rne(__fmul_rn(a[8 + 2 * j], sa.mult), __fmul_rn(a[9 + 2 * j], sa.mult)) << (8 * j);
                        cb0 |= e2m1x2_rne(__fmul_rn(b[2 * j], sb.mult), __fmul_rn(b[2 * j + 1], sb.mult)) << (8 * j);
                        cb1 |= e2m1x2_rne(__fmul_rn(b[8 + 2 * j], sb.mult), __fmul_rn(b[9 + 2 * j], sb.mult)) << (8 * j);
                    }
                }
                const int cl = lane * 8 + 2 * q;  // local column of `a`; `b` is cl + 1
                *reinterpret_cast<uint2*>(s_codes + cl * 32 + warp * 8) = make_uint2(ca0, ca1);
                *reinterpret_cast<uint2*>(s_codes + (cl + 1) * 32 + warp * 8) = make_uint2(cb0, cb1);
                s_scales[cl * 4 + warp] = grp_ok ? (uint8_t)sa.code : (uint8_t)0;
                s_scales[(cl + 1) * 4 + warp] = grp_ok ? (uint8_t)sb.code : (uint8_t)0;
            }
            __syncthreads();
            // write: form row = column c, K segment = this tile's rows
            const int64_t rbase = tr * kTileRows;
            const int64_t cbase = tc * kTileCols;
            const int64_t rem_groups = (rows - rbase) >> 4;
            const int ngroups = rem_groups < 4 ? (int)rem_groups : 4;
            const int64_t kbytes = rows >> 1;  // bytes per form row
            if ((rows & 31) == 0) {
                // 16-byte chunks: 256 columns x 2 chunks (ngroups is even unless the tile is ragged)
                for (int q = threadIdx.x; q < kTileCols * 2; q += kQuantThreads) {
                    const int cl = q >> 1, half = q & 1;
                    if (cbase + cl < cols && 2 * half < ngroups)
                        *reinterpret_cast<uint4*>(p.codes_col + (cbase + cl) * kbytes + (rbase >> 1) + half * 16) =
                            *reinterpret_cast<const uint4*>(s_codes + cl * 32 + half * 16);
                }
            } else {
                for (int q = threadIdx.x; q < kTileCols * 4; q += kQuantThreads) {
                    const int cl = q >> 2, g = q & 3;
                    if (cbase + cl < cols && g < ngroups)
                        *reinterpret_cast<uint2*>(p.codes_col + (cbase + cl) * kbytes + (rbase >> 1) + g * 8) =
                            *reinterpret_cast<const uint2*>(s_codes + cl * 32 + g * 8);
                }
            }
            for (int cl = threadIdx.x; cl < kTileCols; cl += kQuantThreads) {
                if (cbase + cl < cols)
                    *reinterpret_cast<uint32_t*>(p.scales_col + scale_offset(cbase + cl, rbase >> 4, p.nkt_col)) =
                        *reinterpret_cast<const uint32_t*>(s_scales + cl * 4);
            }
            __syncthreads();
        }
    }
}

// ---------------------------------------------------------------------------------------
// K5: transposed layout of a 16x16 form without requantizing.  One thread per 16x16 tile:
// 16 x 8-byte rows in, nibble transpose in registers, 16 x 8-byte rows out.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) transpose_2d_kernel(const uint8_t* __restrict__ codes,
                                                           const uint8_t* __restrict__ tiles, int64_t R,
                                                           int64_t K, uint8_t* __restrict__ codes_t,
                                                           uint8_t* __restrict__ scales_t,
                                                           uint8_t* __restrict__ tiles_t, int64_t nkt_t,
                                                           const float* __restrict__ st_in,
                                                           float* __restrict__ st_out) {
    const int64_t tr_n = R >> 4, tc_n = K >> 4;
    const int64_t total = tr_n * tc_n;
    if (blockIdx.x == 0 && threadIdx.x == 0) *st_out = *st_in;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
        const int64_t a = t / tc_n, b = t - a * tc_n;  // tile (row tile a, k tile b)
        uint64_t in[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            in[i] = *reinterpret_cast<const uint64_t*>(codes + ((a << 4) + i) * (K >> 1) + (b << 3));
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            uint64_t o = 0;
#pragma unroll
            for (int i = 0; i < 16; ++i) o |= ((in[i] >> (4 * j)) & 15ull) << (4 * i);
            *reinterpret_cast<uint64_t*>(codes_t + ((b << 4) + j) * (R >> 1) + (a << 3)) = o;
        }
        const uint8_t s = tiles[a * tc_n + b];
        if (tiles_t) tiles_t[b * tr_n + a] = s;
#pragma unroll
        for (int j = 0; j < 16; ++j) scales_t[scale_offset((b << 4) + j, a, nkt_t)] = s;
    }
}

// ---------------------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------------------
static int grid_for(int64_t work_items, int threads, int per_sm) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t want = (work_items + threads - 1) / threads;
    int64_t cap = (int64_t)sms * per_sm;
    if (want < 1) want = 1;
    return (int)(want < cap ? want : cap);
}

cudaError_t launch_amax_plain(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, uint32_t* amax,
                              uint32_t* flags, cudaStream_t s) {
    const int64_t chunks = rows * (cols >> 3);
    if (chunks == 0) return cudaSuccess;
    amax_plain_kernel<<<grid_for(chunks, 256, 8), 256, 0, s>>>(x, rows, cols, ld, amax, flags);
    return cudaGetLastError();
}

cudaError_t launch_amax_rht(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, uint32_t signs,
                            uint32_t* amax_plain, uint32_t* amax_rht, uint32_t* flags, cudaStream_t s) {
    const int64_t units = (rows >> 4) * (cols >> 3);
    if (units == 0) return cudaSuccess;
    amax_rht_kernel<<<grid_for(units, 256, 2), 256, 0, s>>>(x, rows, cols, ld, signs, amax_plain, amax_rht,
                                                           flags);
    return cudaGetLastError();
}

cudaError_t launch_quantize_tiles(const QuantParams& p, cudaStream_t s) {
    const int64_t ntiles = ((p.rows + kTileRows - 1) / kTileRows) * ((p.cols + kTileCols - 1) / kTileCols);
    if (ntiles == 0) return cudaSuccess;
    const bool row = p.codes_row != nullptr, col = p.codes_col != nullptr;
    const int grid = grid_for(ntiles * kQuantThreads, kQuantThreads, 4);
    if (row && col) quantize_tile_kernel<true, true><<<grid, kQuantThreads, 0, s>>>(p);
    else if (row) quantize_tile_kernel<true, false><<<grid, kQuantThreads, 0, s>>>(p);
    else if (col) quantize_tile_kernel<false, true><<<grid, kQuantThreads, 0, s>>>(p);
    else return cudaErrorInvalidValue;
    return cudaGetLastError();
}

cudaError_t launch_transpose_2d(const uint8_t* codes, const uint8_t* tiles, int64_t R, int64_t K, uint8_t* codes_t,
                                uint8_t* scales_t, uint8_t* tiles_t, const float* st_in, float* st_out,
                                cudaStream_t s) {
    const int64_t total = (R >> 4) * (K >> 4);
    if (total == 0) return cudaSuccess;
    const int64_t nkt_t = ((R >> 4) + 3) >> 2;
    transpose_2d_kernel<<<grid_for(total, 256, 8), 256, 0, s>>>(codes, tiles, R, K, codes_t, scales_t, tiles_t,
                                                               nkt_t, st_in, st_out);
    return cudaGetLastError();
}

}  // namespace nvfp4
