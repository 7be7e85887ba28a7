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
//      magnitude order is the integer order of its low 15 bits), or in fp32 where the pass
//      widens the values for the RHT anyway; one atomicMax per CTA on the fp32 bit pattern
//      (non-negative floats order like unsigned ints, and max does not depend on the order of
//      the reduction).
//   2. quantize (quantize_tile_kernel): persistent CTAs take 64 x 256 tiles of x by TMA into
//      shared memory and emit from one read
//        - the ROW form (K = columns): a 1x16 block is a lane pair, one shuffle for its amax;
//          each lane writes 4 code bytes per row (a warp writes 128 contiguous bytes);
//        - the COL form (K = rows, the transposed wgrad/dgrad operand): a 1x16 block is 16
//          values down one column of the tile, optionally rotated by the 16-point butterfly;
//          codes and scales are staged in shared memory and leave as contiguous row segments.
//      16x16 tiles (weights) share one scale between both forms.  The pass walks the tiles in
//      reverse order of the amax pass so its first wave reads what the amax pass left in L2.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
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
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    uint32_t m = 0;
    if (ld == cols) {
        // contiguous rows: one flat array of 16-byte chunks, four loads in flight per iteration
        const int64_t total = rows * cpr;
        int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
        for (; c + 3 * stride < total; c += 4 * stride) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] = ldg_stream(x + ((c + u * stride) << 3));
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                m = mag_max2(m, v[u].x);
                m = mag_max2(m, v[u].y);
                m = mag_max2(m, v[u].z);
                m = mag_max2(m, v[u].w);
            }
        }
        for (; c < total; c += stride) {
            const uint4 v = ldg_stream(x + (c << 3));
            m = mag_max2(mag_max2(mag_max2(mag_max2(m, v.x), v.y), v.z), v.w);
        }
    }
    GridWalk w((int64_t)blockIdx.x * blockDim.x + threadIdx.x, stride, cpr);
    if (ld == cols) w.r = rows;   // done above
    // four independent loads in flight per iteration
    while (w.r < rows) {
        uint4 v[4];
        bool ok[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            ok[u] = w.r < rows;
            v[u] = ok[u] ? ldg_stream(x + w.r * ld + (w.k << 3)) : make_uint4(0, 0, 0, 0);
            w.next();
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            m = mag_max2(m, v[u].x);
            m = mag_max2(m, v[u].y);
            m = mag_max2(m, v[u].z);
            m = mag_max2(m, v[u].w);
        }
    }
    uint32_t mag = max(m & 0xFFFFu, m >> 16);
    if (mag >= 0x7F80u) atomicOr(flags, kFlagNonFinite);  // Inf (0x7F80) or NaN
    block_atomic_max(mag << 16, amax_bits, red);
}

// ---------------------------------------------------------------------------------------
// pass 1b: plain amax and amax of the 16-point RHT along rows (one read).  A thread takes a
// 16-row x 2-column patch (16 four-byte loads; a warp reads 128 contiguous bytes per row), the
// column pair transformed as f32x2 pairs.  Few registers per thread keep many patches in flight.
// The plain amax is a three-input fp32 max over the widened values that propagates NaN (the sign
// flips do not change magnitudes); the butterfly's final 1/4 is applied once, to the max.
// rows % 16 == 0, cols % 2 == 0.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) amax_rht_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t cols,
                                                       int64_t ld, const SignMasks sm,
                                                       uint32_t* __restrict__ amax_plain_bits,
                                                       uint32_t* __restrict__ amax_rht_bits,
                                                       uint32_t* __restrict__ flags) {
    __shared__ uint32_t red[8];
    const int64_t cpr = cols >> 1;
    const int64_t groups = rows >> 4;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    float mp = 0.0f, mr = 0.0f;
    for (GridWalk w((int64_t)blockIdx.x * blockDim.x + threadIdx.x, stride, cpr); w.r < groups; w.next()) {
        const uint16_t* base = x + (w.r << 4) * ld + (w.k << 1);
        uint32_t v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v[i]) : "l"(base + i * ld));
        uint64_t f[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            f[i] = bf16x2_to_f2(v[i] ^ sm.m[i]);
            float a0, a1;
            f2_split(f[i], a0, a1);
            asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(mp) : "f"(mp), "f"(fabsf(a0)), "f"(fabsf(a1)));
        }
        // the butterfly without its final 1/4: RN(x / 4) is monotonic, so the max of the scaled
        // outputs is the scaled max
#pragma unroll
        for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                if (i & h) continue;
                const uint64_t a = f[i], b = f[i + h];
                f[i] = f2_add(a, b);
                f[i + h] = f2_sub(a, b);
            }
        }
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
            float a0, a1, b0, b1;
            f2_split(f[i], a0, a1);
            f2_split(f[i + 1], b0, b1);
            mr = max3_abs(max3_abs(mr, a0, a1), b0, b1);
        }
    }
    mr = __fmul_rn(mr, 0.25f);
    if (!(mp < __int_as_float(0x7F800000)) || !(mr < __int_as_float(0x7F800000))) atomicOr(flags, kFlagNonFinite);
    block_atomic_max(__float_as_uint(mp), amax_plain_bits, red);
    block_atomic_max(__float_as_uint(mr), amax_rht_bits, red);
}

// ---------------------------------------------------------------------------------------
// pass 2: the tile quantizer.
//
// A persistent CTA of 256 threads walks 64-row x 256-column tiles (in reverse order of the
// amax pass).  Each tile is brought into shared memory by one 2D TMA copy (double-buffered:
// the next tile's copy is in flight while this one is processed) and then consumed in phases
// whose thread mappings each suit one job:
//   T  (16x16) the tile scales: 4 threads per 16x16 tile, two shuffles;
//   R  (ROW form) one thread per 1x16 block: two 16-byte shared loads, the block scale, the 8
//      element pairs scaled as f32x2, 8 code bytes per store; lanes 4a..4a+3 hold four
//      consecutive blocks of a row, whose scales leave as one 32-bit store;
//   C  (COL form) one thread per (column pair, 16-row group): 16 four-byte shared loads give
//      both columns down the group, which stay paired through the optional 16-point RHT, the
//      block amax and the scaling; codes are staged in shared memory;
//   S  (COL form) the staged codes and scales leave as 16-byte (or 8-byte) row segments.
// The rounding mode is a template parameter (one mode per call).  Under SR the Philox fields of
// a block are drawn in place (the fields of a form element are indexed by its position in the
// form, so a COL block's 16 elements are two whole Philox calls), the values are rounded onto the
// E2M1 grid as exact fp32 numbers (e2m1_sr_values), and both modes then encode with the same
// hardware RNE conversion.
// Per-CTA tables hold r_b = S_enc / dec(c) for the 127 finite E4M3 codes (one IEEE division
// each, identical to dividing per block).
// ---------------------------------------------------------------------------------------
constexpr int kTileRows = 64;
constexpr int kTileCols = 256;
constexpr int kQuantThreads = 256;
constexpr int kTileBytes = kTileRows * kTileCols * 2;        // 32 KiB of bf16
// [group][column] x 8 bytes, each group padded by 32 bytes: the S phase's lanes read two groups at
// once (2 apart), which then sit 64 bytes apart in the banks instead of on the same ones
constexpr int kCodeGroupBytes = kTileCols * 8 + 32;
constexpr int kStageCodeBytes = 4 * kCodeGroupBytes;
constexpr int kStageScaleBytes = 4 * kTileCols;              // [group][column]

struct QuantSmem {
    // offsets into the dynamic shared memory (all 128-byte aligned)
    static constexpr int x0 = 0;
    static constexpr int x1 = kTileBytes;
    static constexpr int codes = 2 * kTileBytes;
    static constexpr int scales = codes + kStageCodeBytes;
    static constexpr int mult_row = scales + kStageScaleBytes;   // 128 floats
    static constexpr int mult_col = mult_row + 512;              // 128 floats
    static constexpr int tile_code = mult_col + 512;             // 64 bytes
    static constexpr int tile_mult = tile_code + 128;            // 64 floats
    static constexpr int bars = tile_mult + 256;                 // 2 mbarriers + abort flag
    static constexpr int bytes = bars + 128;
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ bool q_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// bounded wait for a TMA tile: false once about `budget_ns` has passed (counted in SM cycles, 2
// per nanosecond; the counter is read only after a burst of polls)
__device__ __forceinline__ bool q_wait(uint32_t bar, uint32_t parity, uint64_t budget_ns) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
        if (q_try_wait(bar, parity)) return true;
    uint64_t t0;
    asm volatile("mov.u64 %0, %%clock64;" : "=l"(t0));
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (q_try_wait(bar, parity)) return true;
        uint64_t t;
        asm volatile("mov.u64 %0, %%clock64;" : "=l"(t));
        if (t - t0 > 2 * budget_ns) return false;
    }
}

__device__ __forceinline__ void q_load_tile(uint32_t dst, const CUtensorMap* map, int32_t col, int32_t row, uint32_t bar) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"((uint32_t)kTileBytes)
                 : "memory");
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(col), "r"(row), "r"(bar)
        : "memory");
}

__device__ __forceinline__ uint32_t e4m3_of_amax(float amax_b, float s_enc) {
    return e4m3_rne_sat(__fmul_rn(__fdiv_rn(amax_b, 6.0f), s_enc));
}

// Philox4x32-10 of counter (g_lo, g_hi, stream, 0) with the round keys taken from the kernel's
// parameters (constant-bank operands: no registers held for them)
__device__ __forceinline__ U4 sr_words_p(const QuantParams& p, uint32_t stream_id, uint64_t g) {
    uint32_t c0 = (uint32_t)g, c1 = (uint32_t)(g >> 32), c2 = stream_id, c3 = 0u;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ p.key0[r], n2 = (uint32_t)(p0 >> 32) ^ c3 ^ p.key1[r];
        c1 = (uint32_t)p1;
        c3 = (uint32_t)p0;
        c0 = n0;
        c2 = n2;
    }
    return U4{c0, c1, c2, c3};
}

template <bool ROW, bool COL, bool SR>
__global__ void __launch_bounds__(kQuantThreads, 3) quantize_tile_kernel(const __grid_constant__ CUtensorMap tmx,
                                                                     const __grid_constant__ QuantParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x;
    float* s_mult_row = reinterpret_cast<float*>(smem + QuantSmem::mult_row);
    float* s_mult_col = reinterpret_cast<float*>(smem + QuantSmem::mult_col);
    uint8_t* s_tile_code = smem + QuantSmem::tile_code;
    float* s_tile_mult = reinterpret_cast<float*>(smem + QuantSmem::tile_mult);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + QuantSmem::bars);
    volatile uint32_t* s_abort = reinterpret_cast<volatile uint32_t*>(smem + QuantSmem::bars + 16);
    uint8_t* s_codes = smem + QuantSmem::codes;
    uint8_t* s_scales = smem + QuantSmem::scales;

    const int64_t rows = p.rows, cols = p.cols;
    const int64_t ntr = (rows + kTileRows - 1) / kTileRows;
    const int64_t ntc = (cols + kTileCols - 1) / kTileCols;
    const int64_t ntiles = ntr * ntc;
    constexpr bool sr_row = ROW && SR, sr_col = COL && SR;
    const bool rht = COL && p.rht_col, b16 = p.block16 != 0;

    const float senc_r = encode_scale(__uint_as_float(ROW ? *p.amax_row : 0u));
    const float senc_c = encode_scale(__uint_as_float(COL ? *p.amax_col : 0u));
    if (blockIdx.x == 0 && tid == 0) {
        if (ROW) *p.st_row = decode_scale(__uint_as_float(*p.amax_row));
        if (COL) *p.st_col = decode_scale(__uint_as_float(*p.amax_col));
    }
    if (tid < 128) {
        const uint32_t c = (uint32_t)tid;
        if (ROW) s_mult_row[c] = (c == 0 || c == 127) ? 0.0f : __fdiv_rn(senc_r, e4m3_decode(c));
        if (COL) s_mult_col[c] = (c == 0 || c == 127) ? 0.0f : __fdiv_rn(senc_c, e4m3_decode(c));
    }
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(&bars[0])) : "memory");
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(&bars[1])) : "memory");
        *s_abort = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    int64_t it = blockIdx.x;
    auto tile_rc = [&](int64_t i, int64_t& tr, int64_t& tc) {
        const int64_t t = ntiles - 1 - i;
        tr = t / ntc;
        tc = t - tr * ntc;
    };
    if (tid == 0 && it < ntiles) {
        int64_t tr, tc;
        tile_rc(it, tr, tc);
        q_load_tile(smem_addr(smem + QuantSmem::x0), &tmx, (int32_t)(tc * kTileCols), (int32_t)(tr * kTileRows),
                    smem_addr(&bars[0]));
    }
    int issued = (it < ntiles) ? 1 : 0, consumed = 0;

    for (int local = 0; it < ntiles; it += gridDim.x, ++local) {
        const int buf = local & 1;
        int64_t tr, tc;
        tile_rc(it, tr, tc);
        // prefetch the next tile into the other buffer (freed by the previous iteration's sync)
        if (tid == 0 && it + gridDim.x < ntiles) {
            int64_t nr, nc;
            tile_rc(it + gridDim.x, nr, nc);
            q_load_tile(smem_addr(smem + (buf ? QuantSmem::x0 : QuantSmem::x1)), &tmx, (int32_t)(nc * kTileCols),
                        (int32_t)(nr * kTileRows), smem_addr(&bars[buf ^ 1]));
            ++issued;
        }
        if (!q_wait(smem_addr(&bars[buf]), (uint32_t)(local >> 1) & 1u, 2000000000ull)) *s_abort = 1u;
        __syncthreads();
        if (*s_abort) {
            if (tid == 0) atomicOr(p.flags, kFlagTimeout);
            break;
        }
        ++consumed;
        const uint16_t* sx = reinterpret_cast<const uint16_t*>(smem + (buf ? QuantSmem::x1 : QuantSmem::x0));
        const int64_t r_base = tr * kTileRows, c_base = tc * kTileCols;

        // ---- T: 16x16 tile scales ------------------------------------------------------------
        if (b16) {
            // lane = (row quarter q, tile cgl of the warp's 8): the 8 lanes of a quarter-warp read 8
            // different 16-byte bank groups (lanes 4..7 of each group read their second half first)
            const int lane = tid & 31, wq = tid >> 5;
            const int cgl = lane & 7, q = lane >> 3;
            const int g = wq >> 1, cg = ((wq & 1) << 3) + cgl;
            const int tile = (g << 4) + cg;
            const int hf = (cgl >> 2) & 1;
            uint32_t m = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint16_t* rowp = sx + (g * 16 + q * 4 + i) * kTileCols + cg * 16;
                const uint4 a = *reinterpret_cast<const uint4*>(rowp + 8 * hf);
                const uint4 b = *reinterpret_cast<const uint4*>(rowp + 8 * (hf ^ 1));
                m = mag_max2(m, a.x); m = mag_max2(m, a.y); m = mag_max2(m, a.z); m = mag_max2(m, a.w);
                m = mag_max2(m, b.x); m = mag_max2(m, b.y); m = mag_max2(m, b.z); m = mag_max2(m, b.w);
            }
            m = max(m & 0xFFFFu, m >> 16);
            m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 8));
            m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 16));
            const uint32_t code = e4m3_of_amax(__uint_as_float(m << 16), ROW ? senc_r : senc_c);
            if (q == 0) {
                s_tile_code[tile] = (uint8_t)code;
                s_tile_mult[tile] = (ROW ? s_mult_row : s_mult_col)[code];
                const int64_t gr = r_base + g * 16, gc = c_base + cg * 16;
                if (gr < rows && gc < cols) {
                    if (ROW && p.tiles_row) p.tiles_row[(gr >> 4) * (cols >> 4) + (gc >> 4)] = (uint8_t)code;
                    if (COL && p.tiles_col) p.tiles_col[(gc >> 4) * (rows >> 4) + (gr >> 4)] = (uint8_t)code;
                }
            }
            __syncthreads();
        }

        // ---- R: the ROW form, one thread per 1x16 block ----------------------------------------
        // A warp covers two tile rows (16 blocks each); lanes 4a..4a+3 hold four consecutive
        // blocks of one row, whose scales leave as one 32-bit word.
        if (ROW) {
#pragma unroll
            for (int j = tid; j < kTileRows * (kTileCols / 16); j += kQuantThreads) {
                const int r = j >> 4, b = j & 15;
                const int64_t gr = r_base + r, gc = c_base + b * 16;
                // without SR, lanes with (b >> 2) odd read their block's second half first, so that the
                // 8 lanes of a quarter-warp hit 8 different 16-byte bank groups; the two code words are
                // put back in order at the store (under SR the swap costs more than it saves)
                const int hf = SR ? 0 : (b >> 2) & 1;
                const uint4 v0 = *reinterpret_cast<const uint4*>(sx + r * kTileCols + b * 16 + 8 * hf);
                const uint4 v1 = *reinterpret_cast<const uint4*>(sx + r * kTileCols + b * 16 + 8 * (hf ^ 1));
                const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                uint32_t code;
                float mult;
                if (b16) {
                    const int tile = ((r >> 4) << 4) + b;
                    code = s_tile_code[tile];
                    mult = s_tile_mult[tile];
                } else {
                    uint32_t m = 0;
#pragma unroll
                    for (int q = 0; q < 8; ++q) m = mag_max2(m, w[q]);
                    m = max(m & 0xFFFFu, m >> 16);
                    code = e4m3_of_amax(__uint_as_float(m << 16), senc_r);
                    mult = s_mult_row[code];
                }
                const uint64_t mm = f2(mult, mult);
                uint64_t uv[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) uv[q] = f2_mul(bf16x2_to_f2(w[q]), mm);
                if (sr_row) {
                    const uint64_t g0 = ((uint64_t)(p.row_offset + gr) * (uint64_t)cols + (uint64_t)gc) >> 3;
                    const U4 ra = sr_words_p(p, p.stream_row, g0);
                    const U4 rb = sr_words_p(p, p.stream_row, g0 + 1);
                    const uint32_t rr[8] = {ra.x, ra.y, ra.z, ra.w, rb.x, rb.y, rb.z, rb.w};
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        uv[q] = e2m1_sr_values(uv[q], sr_field(rr[q], false), sr_field(rr[q], true));
                }
                uint32_t sw = code | (__shfl_down_sync(0xFFFFFFFFu, code, 1) << 8);
                sw |= __shfl_down_sync(0xFFFFFFFFu, sw, 2) << 16;
                if (gr < rows && gc < cols) {
                    const uint32_t c0 = e2m1x8_word(uv[0], uv[1], uv[2], uv[3]), c1 = e2m1x8_word(uv[4], uv[5], uv[6], uv[7]);
                    *reinterpret_cast<uint2*>(p.codes_row + gr * (cols >> 1) + (gc >> 1)) =
                        make_uint2(hf ? c1 : c0, hf ? c0 : c1);
                    if ((b & 3) == 0) {
                        // blocks past `cols` are padding and must read 0
                        const int64_t kb = gc >> 4;
                        const int64_t nv64 = (cols >> 4) - kb;
                        const int nvalid = nv64 < 4 ? (int)nv64 : 4;
                        const uint32_t keep = nvalid >= 4 ? 0xFFFFFFFFu : ((1u << (8 * nvalid)) - 1u);
                        *reinterpret_cast<uint32_t*>(p.scales_row + scale_offset(gr, kb, p.nkt_row)) = sw & keep;
                    }
                }
            }
        }

        // ---- C: the COL form, one thread per (column pair, 16-row group) -----------------------
        // The two columns' 16 values arrive as 16 bf16 pairs (one 32-bit shared load per row) and
        // stay paired through the RHT and the scaling (f32x2 arithmetic).  The SR fields of a form
        // element are indexed by its position in the form, so each column's 16 elements are two
        // whole Philox calls.
        if (COL) {
#pragma unroll
            for (int j = tid; j < 4 * (kTileCols / 2); j += kQuantThreads) {
                const int cp = j & (kTileCols / 2 - 1), g = j >> 7;   // a warp covers 64 columns of one group
                const int c = 2 * cp;
                uint64_t v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    uint32_t w = *reinterpret_cast<const uint32_t*>(sx + (g * 16 + i) * kTileCols + c);
                    if (rht) w ^= p.sign_mask2[i];
                    v[i] = bf16x2_to_f2(w);
                }
                if (rht) rht16_pairs(v);
                uint32_t code0, code1;
                float mult0, mult1;
                if (b16) {
                    const int tile = (g << 4) + (c >> 4);
                    code0 = code1 = s_tile_code[tile];
                    mult0 = mult1 = s_tile_mult[tile];
                } else {
                    float m0 = 0.0f, m1 = 0.0f;
#pragma unroll
                    for (int i = 0; i < 16; i += 2) {
                        float a0, a1, b0, b1;
                        f2_split(v[i], a0, a1);
                        f2_split(v[i + 1], b0, b1);
                        m0 = max3_abs(m0, a0, b0);
                        m1 = max3_abs(m1, a1, b1);
                    }
                    code0 = e4m3_of_amax(m0, senc_c);
                    code1 = e4m3_of_amax(m1, senc_c);
                    mult0 = s_mult_col[code0];
                    mult1 = s_mult_col[code1];
                }
                const uint64_t mm = f2(mult0, mult1);
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = f2_mul(v[i], mm);
                uint32_t out[4];   // column c: out[0..1], column c + 1: out[2..3]
                if (sr_col) {
                    // form element (column c, row r) has index c * rows_total + row_offset + r; the
                    // block's first row is a multiple of 16, so its 16 fields are Philox calls i0/8, i0/8 + 1
                    const uint64_t g0 = ((uint64_t)(c_base + c) * (uint64_t)p.rows_total +
                                         (uint64_t)(p.row_offset + r_base + g * 16)) >> 3;
                    const uint64_t g1 = g0 + ((uint64_t)p.rows_total >> 3);   // column c + 1
#pragma unroll
                    for (int h = 0; h < 2; ++h) {   // rows 8h .. 8h + 7: one Philox call per column
                        const U4 a = sr_words_p(p, p.stream_col, g0 + h), b = sr_words_p(p, p.stream_col, g1 + h);
                        const uint32_t ra[4] = {a.x, a.y, a.z, a.w}, rb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            v[8 * h + i] = e2m1_sr_values(v[8 * h + i], sr_field(ra[i >> 1], i & 1),
                                                          sr_field(rb[i >> 1], i & 1));
                    }
                }
                {
                    float e0[16], e1[16];   // column c and column c + 1, rows 0..15
#pragma unroll
                    for (int i = 0; i < 16; ++i) f2_split(v[i], e0[i], e1[i]);
                    out[0] = e2m1x8_word(e0[0], e0[1], e0[2], e0[3], e0[4], e0[5], e0[6], e0[7]);
                    out[1] = e2m1x8_word(e0[8], e0[9], e0[10], e0[11], e0[12], e0[13], e0[14], e0[15]);
                    out[2] = e2m1x8_word(e1[0], e1[1], e1[2], e1[3], e1[4], e1[5], e1[6], e1[7]);
                    out[3] = e2m1x8_word(e1[8], e1[9], e1[10], e1[11], e1[12], e1[13], e1[14], e1[15]);
                }
                const bool grp_ok = r_base + g * 16 < rows;
                *reinterpret_cast<uint4*>(s_codes + g * kCodeGroupBytes + c * 8) = make_uint4(out[0], out[1], out[2], out[3]);
                *reinterpret_cast<uint16_t*>(s_scales + g * kTileCols + c) = grp_ok ? (uint16_t)(code0 | (code1 << 8)) : (uint16_t)0;
            }
            __syncthreads();
            // ---- S: staged COL codes and scales to global memory ---------------------------------
            const int64_t rem = (rows - r_base) >> 4;
            const int ngroups = rem < 4 ? (int)rem : 4;
            const int64_t kbytes = rows >> 1;
            if ((rows & 31) == 0) {
#pragma unroll 1
                for (int j = tid; j < 2 * kTileCols; j += kQuantThreads) {
                    const int c = j >> 1, half = j & 1;
                    if (c_base + c < cols && 2 * half < ngroups) {
                        const uint2 lo = *reinterpret_cast<const uint2*>(s_codes + (2 * half) * kCodeGroupBytes + c * 8);
                        const uint2 hi = *reinterpret_cast<const uint2*>(s_codes + (2 * half + 1) * kCodeGroupBytes + c * 8);
                        *reinterpret_cast<uint4*>(p.codes_col + (c_base + c) * kbytes + (r_base >> 1) + half * 16) =
                            make_uint4(lo.x, lo.y, hi.x, hi.y);
                    }
                }
            } else {
#pragma unroll 1
                for (int j = tid; j < 4 * kTileCols; j += kQuantThreads) {
                    const int c = j >> 2, g = j & 3;
                    if (c_base + c < cols && g < ngroups)
                        *reinterpret_cast<uint2*>(p.codes_col + (c_base + c) * kbytes + (r_base >> 1) + g * 8) =
                            *reinterpret_cast<const uint2*>(s_codes + g * kCodeGroupBytes + c * 8);
                }
            }
            for (int c = tid; c < kTileCols; c += kQuantThreads) {
                if (c_base + c < cols) {
                    const uint32_t w = (uint32_t)s_scales[c] | ((uint32_t)s_scales[kTileCols + c] << 8) |
                                       ((uint32_t)s_scales[2 * kTileCols + c] << 16) |
                                       ((uint32_t)s_scales[3 * kTileCols + c] << 24);
                    *reinterpret_cast<uint32_t*>(p.scales_col + scale_offset(c_base + c, r_base >> 4, p.nkt_col)) = w;
                }
            }
        }
        __syncthreads();   // the buffer and the staging areas are free for the next tile
    }
    // copies issued but never consumed (only after a timeout) must land before the CTA exits
    if (tid == 0) {
        for (int k = consumed; k < issued; ++k) q_wait(smem_addr(&bars[k & 1]), (uint32_t)(k >> 1) & 1u, 2000000000ull);
    }
}

// ---------------------------------------------------------------------------------------
// MXFP4, the pages' comparison format (gist.science 2.A): blocks of 32 elements along K, one
// UE8M0 scale 2^E per block with E = floor(log2 amax_b) - 2 (2 = the largest E2M1 exponent;
// stored as E + 127, clamped to [0, 254]; an all-zero block gets 0), no tensor scale and so no
// amax pass.  Elements u = v * 2^-E (one exact power-of-two product, rounded only if it lands
// below the normal range) go through the same E2M1 encoders as NVFP4, RNE or SR; SR fields are
// indexed by the element's position in the form.  The same TMA-fed persistent tile walk as the
// NVFP4 quantizer, one form or both forms from one read of each tile:
//   ROW form: one thread per 1x32 block (four 16-byte shared loads), 16 code bytes per store;
//   COL form: one thread per (column pair, 32-row group): the 32 bf16 pairs give both columns'
//             block maxima by packed integer max, then the codes are staged and leave as rows.
// ---------------------------------------------------------------------------------------
// UE8M0 code of a block whose largest magnitude has bf16 bits m (sign cleared)
__device__ __forceinline__ uint32_t ue8m0_of_mag(uint32_t m) {
    if (m == 0) return 0u;
    const int e = (int)(m >> 7);
    const int fl = e ? e - 127 : (31 - __clz((int)(m & 0x7Fu))) - 133;   // floor(log2 amax_b)
    return (uint32_t)min(max(fl + 125, 0), 254);
}
// 2^-E = 2^(127 - code), exact (2^-127 is the one subnormal case)
__device__ __forceinline__ float ue8m0_inv(uint32_t code) {
    return __uint_as_float(code == 254u ? 0x00400000u : (254u - code) << 23);
}

__device__ __forceinline__ U4 mx_words(const MxParams& p, uint32_t stream_id, uint64_t g) {
    uint32_t c0 = (uint32_t)g, c1 = (uint32_t)(g >> 32), c2 = stream_id, c3 = 0u;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ p.key0[r], n2 = (uint32_t)(p0 >> 32) ^ c3 ^ p.key1[r];
        c1 = (uint32_t)p1;
        c3 = (uint32_t)p0;
        c0 = n0;
        c2 = n2;
    }
    return U4{c0, c1, c2, c3};
}

template <bool ROWF, bool COLF>
__global__ void __launch_bounds__(kQuantThreads, 3) quantize_mx_kernel(const __grid_constant__ CUtensorMap tmx,
                                                                      const __grid_constant__ MxParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + QuantSmem::bars);
    volatile uint32_t* s_abort = reinterpret_cast<volatile uint32_t*>(smem + QuantSmem::bars + 16);
    uint8_t* s_codes = smem + QuantSmem::codes;
    uint8_t* s_scales = smem + QuantSmem::scales;
    const int64_t rows = p.rows, cols = p.cols;
    const int64_t ntr = (rows + kTileRows - 1) / kTileRows;
    const int64_t ntc = (cols + kTileCols - 1) / kTileCols;
    const int64_t ntiles = ntr * ntc;
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(&bars[0])) : "memory");
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(&bars[1])) : "memory");
        *s_abort = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    int64_t it = blockIdx.x;
    if (tid == 0 && it < ntiles)
        q_load_tile(smem_addr(smem + QuantSmem::x0), &tmx, (int32_t)((it % ntc) * kTileCols), (int32_t)((it / ntc) * kTileRows),
                    smem_addr(&bars[0]));
    int issued = (it < ntiles) ? 1 : 0, consumed = 0;
    for (int local = 0; it < ntiles; it += gridDim.x, ++local) {
        const int buf = local & 1;
        const int64_t tr = it / ntc, tc = it - tr * ntc;
        if (tid == 0 && it + gridDim.x < ntiles) {
            const int64_t n = it + gridDim.x;
            q_load_tile(smem_addr(smem + (buf ? QuantSmem::x0 : QuantSmem::x1)), &tmx, (int32_t)((n % ntc) * kTileCols),
                        (int32_t)((n / ntc) * kTileRows), smem_addr(&bars[buf ^ 1]));
            ++issued;
        }
        if (!q_wait(smem_addr(&bars[buf]), (uint32_t)(local >> 1) & 1u, 2000000000ull)) *s_abort = 1u;
        __syncthreads();
        if (*s_abort) {
            if (tid == 0) atomicOr(p.flags, kFlagTimeout);
            break;
        }
        ++consumed;
        const uint16_t* sx = reinterpret_cast<const uint16_t*>(smem + (buf ? QuantSmem::x1 : QuantSmem::x0));
        const int64_t r_base = tr * kTileRows, c_base = tc * kTileCols;
        if (ROWF) {
            // ---- ROW form: one thread per 1x32 block; lanes 4a..4a+3 hold four blocks of one row
#pragma unroll 1
            for (int j = tid; j < kTileRows * (kTileCols / 32); j += kQuantThreads) {
                const int r = j >> 3, b = j & 7;
                const int64_t gr = r_base + r, gc = c_base + b * 32;
                uint32_t w[16];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 v = *reinterpret_cast<const uint4*>(sx + r * kTileCols + b * 32 + 8 * q);
                    w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
                }
                uint32_t m = 0;
#pragma unroll
                for (int q = 0; q < 16; ++q) m = mag_max2(m, w[q]);
                const uint32_t code = ue8m0_of_mag(max(m & 0xFFFFu, m >> 16));
                const float inv = ue8m0_inv(code);
                const uint64_t mm = f2(inv, inv);
                uint64_t uv[16];   // the 16 pairs after scaling (and SR onto the grid)
                if (p.sr) {
                    const uint64_t g0 = ((uint64_t)gr * (uint64_t)cols + (uint64_t)gc) >> 3;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const U4 rw = mx_words(p, p.stream_id, g0 + c);
                        const uint32_t rr[4] = {rw.x, rw.y, rw.z, rw.w};
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            uv[4 * c + q] = e2m1_sr_values(f2_mul(bf16x2_to_f2(w[4 * c + q]), mm), sr_field(rr[q], false),
                                                           sr_field(rr[q], true));
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 16; ++q) uv[q] = f2_mul(bf16x2_to_f2(w[q]), mm);
                }
                uint32_t sw = code | (__shfl_down_sync(0xFFFFFFFFu, code, 1) << 8);
                sw |= __shfl_down_sync(0xFFFFFFFFu, sw, 2) << 16;
                if (gr < rows && gc < cols) {
                    *reinterpret_cast<uint4*>(p.codes + gr * (cols >> 1) + (gc >> 1)) =
                        make_uint4(e2m1x8_word(uv[0], uv[1], uv[2], uv[3]), e2m1x8_word(uv[4], uv[5], uv[6], uv[7]),
                                   e2m1x8_word(uv[8], uv[9], uv[10], uv[11]), e2m1x8_word(uv[12], uv[13], uv[14], uv[15]));
                    if ((b & 3) == 0) {
                        const int64_t kb = gc >> 5;
                        const int64_t nv64 = (cols >> 5) - kb;
                        const int nvalid = nv64 < 4 ? (int)nv64 : 4;
                        const uint32_t keep = nvalid >= 4 ? 0xFFFFFFFFu : ((1u << (8 * nvalid)) - 1u);
                        *reinterpret_cast<uint32_t*>(p.scales + scale_offset(gr, kb, p.nkt)) = sw & keep;
                    }
                }
            }
        }
        if (COLF) {
            // ---- COL form: one thread per (column pair, 32-row group) -------------------------
            {
                const int cp = tid & (kTileCols / 2 - 1), g = tid >> 7;
                const int c = 2 * cp;
                uint32_t w[32];
                uint32_t m = 0;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    w[i] = *reinterpret_cast<const uint32_t*>(sx + (g * 32 + i) * kTileCols + c);
                    m = mag_max2(m, w[i]);
                }
                const uint32_t code0 = ue8m0_of_mag(m & 0xFFFFu), code1 = ue8m0_of_mag(m >> 16);
                const uint64_t mm = f2(ue8m0_inv(code0), ue8m0_inv(code1));
                uint32_t out[8];   // column c: out[0..3], column c + 1: out[4..7]
                if (p.sr) {
                    const uint64_t g0 = ((uint64_t)(c_base + c) * (uint64_t)rows + (uint64_t)(r_base + g * 32)) >> 3;
                    const uint64_t g1 = g0 + ((uint64_t)rows >> 3);
#pragma unroll
                    for (int h = 0; h < 4; ++h) {   // rows 8h .. 8h + 7: one Philox call per column
                        const U4 a = mx_words(p, p.stream_col, g0 + h), bw = mx_words(p, p.stream_col, g1 + h);
                        const uint32_t ra[4] = {a.x, a.y, a.z, a.w}, rb[4] = {bw.x, bw.y, bw.z, bw.w};
                        uint64_t sv[8];   // row i: the SR values of columns c and c + 1
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            sv[i] = e2m1_sr_values(f2_mul(bf16x2_to_f2(w[8 * h + i]), mm), sr_field(ra[i >> 1], i & 1),
                                                   sr_field(rb[i >> 1], i & 1));
                        float e0[8], e1[8];   // column c and column c + 1, rows 8h .. 8h + 7
#pragma unroll
                        for (int i = 0; i < 8; ++i) f2_split(sv[i], e0[i], e1[i]);
                        out[h] = e2m1x8_word(e0[0], e0[1], e0[2], e0[3], e0[4], e0[5], e0[6], e0[7]);
                        out[4 + h] = e2m1x8_word(e1[0], e1[1], e1[2], e1[3], e1[4], e1[5], e1[6], e1[7]);
                    }
                } else {
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        float e0[8], e1[8];   // column c and column c + 1, rows 8h .. 8h + 7
#pragma unroll
                        for (int i = 0; i < 8; ++i) f2_split(f2_mul(bf16x2_to_f2(w[8 * h + i]), mm), e0[i], e1[i]);
                        out[h] = e2m1x8_word(e0[0], e0[1], e0[2], e0[3], e0[4], e0[5], e0[6], e0[7]);
                        out[4 + h] = e2m1x8_word(e1[0], e1[1], e1[2], e1[3], e1[4], e1[5], e1[6], e1[7]);
                    }
                }
                const bool grp_ok = r_base + g * 32 < rows;
                *reinterpret_cast<uint4*>(s_codes + (g * kTileCols + c) * 16) = make_uint4(out[0], out[1], out[2], out[3]);
                *reinterpret_cast<uint4*>(s_codes + (g * kTileCols + c + 1) * 16) = make_uint4(out[4], out[5], out[6], out[7]);
                *reinterpret_cast<uint16_t*>(s_scales + g * kTileCols + c) = grp_ok ? (uint16_t)(code0 | (code1 << 8)) : (uint16_t)0;
            }
            __syncthreads();
            // staged codes and scales to global memory: per column 16 code bytes and one scale per group
            const int64_t rem = (rows - r_base) >> 5;
            const int ngroups = rem < 2 ? (int)rem : 2;
            const int64_t kbytes = rows >> 1;
#pragma unroll 1
            for (int j = tid; j < 2 * kTileCols; j += kQuantThreads) {
                const int c = j >> 1, g = j & 1;
                if (c_base + c < cols && g < ngroups)
                    *reinterpret_cast<uint4*>(p.codes_col + (c_base + c) * kbytes + (r_base >> 1) + g * 16) =
                        *reinterpret_cast<const uint4*>(s_codes + (g * kTileCols + c) * 16);
            }
            for (int c = tid; c < kTileCols; c += kQuantThreads) {
                if (c_base + c < cols) {
                    uint8_t* dst = p.scales_col + scale_offset(c_base + c, r_base >> 5, p.nkt_col);
                    dst[0] = s_scales[c];
                    if (ngroups > 1) dst[1] = s_scales[kTileCols + c];
                }
            }
        }
        __syncthreads();
    }
    if (tid == 0) {
        for (int k = consumed; k < issued; ++k) q_wait(smem_addr(&bars[k & 1]), (uint32_t)(k >> 1) & 1u, 2000000000ull);
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
// SM count of the current device, looked up once per device
static int q_sm_count() {
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// Resident CTAs per SM of a tile kernel on the current device, with its dynamic shared-memory
// limit raised first; both are per-device facts of the kernel, established once per device
// (`cache` belongs to one kernel instantiation).  0 on a CUDA error.
template <typename Kernel>
static int tile_ctas_per_sm(Kernel kern, int threads, int smem, std::atomic<int> (&cache)[64]) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    const bool cacheable = dev >= 0 && dev < 64;
    if (cacheable) {
        const int n = cache[dev].load(std::memory_order_acquire);
        if (n > 0) return n;
    }
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return 0;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem) != cudaSuccess) return 0;
    if (per_sm < 1) per_sm = 1;
    if (cacheable) cache[dev].store(per_sm, std::memory_order_release);
    return per_sm;
}

static int grid_for(int64_t work_items, int threads, int per_sm) {
    const int sms = q_sm_count();
    int64_t want = (work_items + threads - 1) / threads;
    int64_t cap = (int64_t)sms * per_sm;
    if (want < 1) want = 1;
    return (int)(want < cap ? want : cap);
}

cudaError_t launch_amax_plain(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, uint32_t* amax,
                              uint32_t* flags, cudaStream_t s) {
    const int64_t chunks = rows * (cols >> 3);
    if (chunks == 0) return cudaSuccess;
    amax_plain_kernel<<<grid_for(chunks, 256, 4), 256, 0, s>>>(x, rows, cols, ld, amax, flags);
    return cudaGetLastError();
}

cudaError_t launch_amax_rht(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, uint32_t signs,
                            uint32_t* amax_plain, uint32_t* amax_rht, uint32_t* flags, cudaStream_t s) {
    const int64_t units = (rows >> 4) * (cols >> 1);
    if (units == 0) return cudaSuccess;
    amax_rht_kernel<<<grid_for(units, 256, 4), 256, 0, s>>>(x, rows, cols, ld, sign_masks(signs), amax_plain,
                                                           amax_rht, flags);
    return cudaGetLastError();
}

static PFN_cuTensorMapEncodeTiled_v12000 q_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    return fn;
}

cudaError_t launch_quantize_tiles(const QuantParams& p, cudaStream_t s) {
    const int64_t ntiles = ((p.rows + kTileRows - 1) / kTileRows) * ((p.cols + kTileCols - 1) / kTileCols);
    if (ntiles == 0) return cudaSuccess;
    const bool row = p.codes_row != nullptr, col = p.codes_col != nullptr;
    if (!row && !col) return cudaErrorInvalidValue;
    auto fn = q_encode_fn();
    if (!fn) return cudaErrorInvalidValue;
    CUtensorMap map;
    cuuint64_t dims[2] = {(cuuint64_t)p.cols, (cuuint64_t)p.rows};
    cuuint64_t strides[1] = {(cuuint64_t)(p.ld * 2)};
    cuuint32_t box[2] = {(cuuint32_t)kTileCols, (cuuint32_t)kTileRows};
    cuuint32_t estr[2] = {1u, 1u};
    if (fn(&map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t*>(p.x), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    QuantParams q = p;
    for (int j = 0; j < 16; ++j) q.sign_mask2[j] = ((p.signs >> j) & 1u) ? 0x80008000u : 0u;
    uint32_t k0 = (uint32_t)p.sr_seed, k1 = (uint32_t)(p.sr_seed >> 32);
    for (int r = 0; r < 10; ++r) {   // the Philox4x32-10 key schedule (Salmon et al., SC'11)
        q.key0[r] = k0;
        q.key1[r] = k1;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    const int smem = QuantSmem::bytes;
    const bool sr = (row && p.sr_row) || (col && p.sr_col);   // one rounding mode per call
    void (*kern)(const CUtensorMap, const QuantParams) =
        sr ? (row && col ? quantize_tile_kernel<true, true, true> : row ? quantize_tile_kernel<true, false, true>
                                                                       : quantize_tile_kernel<false, true, true>)
           : (row && col ? quantize_tile_kernel<true, true, false> : row ? quantize_tile_kernel<true, false, false>
                                                                        : quantize_tile_kernel<false, true, false>);
    static std::atomic<int> cache[6][64];   // one per instantiation: (row, col, sr)
    const int which = (sr ? 3 : 0) + (row && col ? 0 : row ? 1 : 2);
    const int per_sm = tile_ctas_per_sm(kern, kQuantThreads, smem, cache[which]);
    if (per_sm < 1) {
        const cudaError_t e = cudaGetLastError();
        return e != cudaSuccess ? e : cudaErrorInvalidValue;
    }
    const int64_t cap = (int64_t)q_sm_count() * per_sm;
    const int grid = (int)(ntiles < cap ? ntiles : cap);
    kern<<<grid, kQuantThreads, smem, s>>>(map, q);
    return cudaGetLastError();
}

cudaError_t launch_quantize_mx(const MxParams& p, bool row_form, bool column_form, uint64_t sr_seed, cudaStream_t s) {
    if (!row_form && !column_form) return cudaErrorInvalidValue;
    const int64_t ntiles = ((p.rows + kTileRows - 1) / kTileRows) * ((p.cols + kTileCols - 1) / kTileCols);
    if (ntiles == 0) return cudaSuccess;
    auto fn = q_encode_fn();
    if (!fn) return cudaErrorInvalidValue;
    CUtensorMap map;
    cuuint64_t dims[2] = {(cuuint64_t)p.cols, (cuuint64_t)p.rows};
    cuuint64_t strides[1] = {(cuuint64_t)(p.ld * 2)};
    cuuint32_t box[2] = {(cuuint32_t)kTileCols, (cuuint32_t)kTileRows};
    cuuint32_t estr[2] = {1u, 1u};
    if (fn(&map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t*>(p.x), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    MxParams q = p;
    uint32_t k0 = (uint32_t)sr_seed, k1 = (uint32_t)(sr_seed >> 32);
    for (int r = 0; r < 10; ++r) {   // the Philox4x32-10 key schedule
        q.key0[r] = k0;
        q.key1[r] = k1;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    void (*kern)(const CUtensorMap, const MxParams) = !column_form ? quantize_mx_kernel<true, false>
                                                      : row_form   ? quantize_mx_kernel<true, true>
                                                                   : quantize_mx_kernel<false, true>;
    static std::atomic<int> cache[3][64];   // row form, column form, both
    const int which = row_form && column_form ? 2 : column_form ? 1 : 0;
    const int per_sm = tile_ctas_per_sm(kern, kQuantThreads, QuantSmem::bytes, cache[which]);
    if (per_sm < 1) {
        const cudaError_t e = cudaGetLastError();
        return e != cudaSuccess ? e : cudaErrorInvalidValue;
    }
    const int64_t cap = (int64_t)q_sm_count() * per_sm;
    kern<<<(int)(ntiles < cap ? ntiles : cap), kQuantThreads, QuantSmem::bytes, s>>>(map, q);
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
