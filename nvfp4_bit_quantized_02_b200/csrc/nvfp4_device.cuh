// nvfp4_device.cuh -- device primitives of the NVFP4 quantization path (sm_100a).
//
// Number formats (gist.science "Pretraining Large Language Models with NVFP4", Technische
// Zusammenfassung 2.A): E2M1 elements, E4M3 block scales, an fp32 tensor scale.  Rounding
// (2.B.4): round-to-nearest-even, or stochastic rounding for gradients.  Rotation (2.B.2): a
// seeded 16-point Random Hadamard Transform.
//
// Every fp32 operation whose result decides a code is written as one IEEE operation with an
// explicit rounding mode (__fdiv_rn / __fmul_rn / __fadd_rn / __fsub_rn, the f32x2 .rn forms, and
// the one round-up add of the stochastic rounding), never contracted or reassociated by the
// compiler, so that codes and scales are reproducible bit for bit.
#pragma once

#include <cstdint>

namespace nvfp4 {

// ---------------------------------------------------------------------------------------
// bf16 unpacking (bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 bits)
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t pair) { return __uint_as_float(pair << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t pair) { return __uint_as_float(pair & 0xFFFF0000u); }

// fp32 -> bf16 bits, round to nearest even (hardware cvt).
__device__ __forceinline__ uint32_t f32x2_to_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// ---------------------------------------------------------------------------------------
// Packed fp32 pairs: sm_100's f32x2 arithmetic performs two independent IEEE round-to-nearest
// operations per instruction, bit-identical to two scalar __fadd_rn / __fsub_rn / __fmul_rn.
// A pair is a 64-bit register {lo, hi}.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2c(float v) { return f2(v, v); }
// the bf16 pair of a 32-bit word (low half = first element) widened to an fp32 pair (exact)
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t w) {
    return f2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
// max(a, |b|, |c|) in one instruction (three-input max of sm_100)
__device__ __forceinline__ float max3_abs(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(fabsf(b)), "f"(fabsf(c)));
    return r;
}

// ---------------------------------------------------------------------------------------
// E2M1 encode, round-to-nearest-even, saturating to +-6, sign kept.  Two values per
// instruction; `lo` lands in bits [0,4), `hi` in bits [4,8).
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t e2m1x2_rne(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
        "cvt.u32.u8 %0, t;\n\t}"
        : "=r"(r)
        : "f"(hi), "f"(lo));
    return r;
}
// Eight values (four pairs) -> one word of codes, pair q in byte q (first value in the low
// nibble).  The four conversions write byte registers that one move packs: no widening of each
// byte and no byte permutes, which the per-pair form above needs to assemble the same word.
__device__ __forceinline__ uint32_t e2m1x8_word(float a0, float a1, float b0, float b1, float c0, float c1, float d0,
                                                float d1) {
    uint32_t r;
    asm("{\n\t.reg .b8 t0, t1, t2, t3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t3, %8, %7;\n\t"
        "mov.b32 %0, {t0, t1, t2, t3};\n\t}"
        : "=r"(r)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1), "f"(d0), "f"(d1));
    return r;
}
// the same from four f32x2 pairs
__device__ __forceinline__ uint32_t e2m1x8_word(uint64_t p0, uint64_t p1, uint64_t p2, uint64_t p3) {
    float a0, a1, b0, b1, c0, c1, d0, d1;
    f2_split(p0, a0, a1);
    f2_split(p1, b0, b1);
    f2_split(p2, c0, c1);
    f2_split(p3, d0, d1);
    return e2m1x8_word(a0, a1, b0, b1, c0, c1, d0, d1);
}

// ---------------------------------------------------------------------------------------
// E2M1 stochastic rounding.  For |u| in [lo, hi) of the grid {0,.5,1,1.5,2,3,4,6} the value
// goes up iff r16 < ceil(((|u| - lo) / (hi - lo)) * 2^16); |u| >= 6 gives 6; sign kept.
// The fraction is read straight from the fp32 bits (all quantities are exact):
//   |u| in [1, 6):   lo keeps the exponent and the top mantissa bit, step = 2^(e-1), so
//                    f * 2^16 = (mantissa & 0x3FFFFF) / 2^6;
//   |u| in [.5, 1):  lo = .5, step = .5, f * 2^16 = mantissa / 2^7;
//   |u| in [0, .5):  lo = 0, step = .5, f * 2^16 = |u| * 2^17 (exact power-of-two scaling).
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t e2m1_sr_threshold(uint32_t a /* |u| bits */) {
    if (a >= 0x3F800000u) return ((a & 0x3FFFFFu) + 63u) >> 6;
    if (a >= 0x3F000000u) return ((a & 0x7FFFFFu) + 127u) >> 7;
    return (uint32_t)ceilf(__fmul_rn(__uint_as_float(a), 131072.0f));
}

// The same decision without computing the threshold, as exact fp32 arithmetic on a pair (two
// elements per f32x2 instruction, on the multiply-add pipe).  With s the grid step of |u|'s cell
// (1/2 below 2, 1 on [2, 4), 2 from 4 up), |u| goes up iff r16 < ceil(f 2^16) with f = (|u| - lo)/s,
// i.e. iff f 2^16 > r16, i.e. iff w = |u| - s r16 / 2^16 > lo; and since w lies in (lo - s, |u|],
// the rounded value is s * ceil(w / s):
//   - s = 2^max(e, 0) / 2 for |u| in [2^e, 2^(e+1)), read from the exponent bits;
//   - w is one fused multiply-add.  It is exact from |u| = 1/2 up (|u| and s r16 / 2^16 are both
//     multiples of |u|'s ulp, and so is w, within |u|'s binade or the one below); below 1/2 it
//     may round but keeps its sign and zero, which is all the step-1/2 ceiling there reads;
//   - the ceiling is one round-up add of 1.5 s 2^23 (whose binade has ulp s), and the subtraction
//     of 1.5 s 2^23 that follows is exact.
// The result is a signed grid value (the sign of u, also for a zero result), 8 where |u| > 6
// rounded up: the hardware RNE conversion to E2M1 then encodes it exactly (8 saturates to 6).
// r_lo / r_hi are the elements' 16-bit fields r16 as fp32 numbers (exact; sr_field).
__device__ __forceinline__ float sr_field(uint32_t word, bool high) {
    // the low (high = false) or the high 16-bit field of a Philox word, converted to fp32 by the
    // integer-to-float unit (which the encode's other instructions leave idle)
    float r;
    if (high)
        asm("{\n\t.reg .u16 a, b;\n\tmov.b32 {a, b}, %1;\n\tcvt.rn.f32.u16 %0, b;\n\t}" : "=f"(r) : "r"(word));
    else
        asm("{\n\t.reg .u16 a, b;\n\tmov.b32 {a, b}, %1;\n\tcvt.rn.f32.u16 %0, a;\n\t}" : "=f"(r) : "r"(word));
    return r;
}
__device__ __forceinline__ uint64_t e2m1_sr_values(uint64_t u, float r_lo, float r_hi) {
    float ul, uh;
    f2_split(u, ul, uh);
    const float el = fmaxf(__uint_as_float(__float_as_uint(ul) & 0x7F800000u), 1.0f);   // 2^max(e, 0)
    const float eh = fmaxf(__uint_as_float(__float_as_uint(uh) & 0x7F800000u), 1.0f);
    const uint64_t nsq = f2_mul(f2(el, eh), f2c(-0x1p-17f));                              // -s / 2^16
    const uint64_t w = f2_fma(nsq, f2(r_lo, r_hi), f2(fabsf(ul), fabsf(uh)));
    const uint64_t m = f2_mul(nsq, f2c(-0x1.8p+39f));                                     // 1.5 s 2^23
    uint64_t t;
    asm("add.rp.f32x2 %0, %1, %2;" : "=l"(t) : "l"(w), "l"(m));
    float vl, vh;
    f2_split(f2_sub(t, m), vl, vh);
    return f2(copysignf(vl, ul), copysignf(vh, uh));
}
// One element: its code in bits [0, 4)
__device__ __forceinline__ uint32_t e2m1_sr(float u, uint32_t r16) {
    const float r = sr_field(r16, false);
    float vl, vh;
    f2_split(e2m1_sr_values(f2(u, u), r, r), vl, vh);
    return e2m1x2_rne(vl, vh) & 15u;
}

// ---------------------------------------------------------------------------------------
// E4M3 ("fn": no infinities, 0x7F = NaN) for non-negative block scales
// ---------------------------------------------------------------------------------------
// Round-to-nearest-even with saturation to 448 (hardware cvt, .satfinite).
__device__ __forceinline__ uint32_t e4m3_rne_sat(float y) {
    uint32_t r;
    asm("{\n\t.reg .b16 t;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\t"
        "cvt.u32.u16 %0, t;\n\t}"
        : "=r"(r)
        : "f"(0.0f), "f"(y));
    return r & 0xFFu;
}

// Value of a non-negative, non-NaN code: m * 2^-9 for exponent field 0, else
// (1 + m/8) * 2^(e-7), assembled directly as fp32 bits.
__device__ __forceinline__ float e4m3_decode(uint32_t c) {
    const uint32_t e = (c >> 3) & 15u, m = c & 7u;
    return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : __fmul_rn((float)m, 0.001953125f);
}

// ---------------------------------------------------------------------------------------
// Tensor-level scales (two-level scaling, 2.A): S_enc = 6*448/amax_t, s_t = amax_t/(6*448),
// one IEEE division each; an all-zero tensor gets 1 and 1.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ float encode_scale(float amax_t) {
    return amax_t > 0.0f ? __fdiv_rn(2688.0f, amax_t) : 1.0f;
}
__device__ __forceinline__ float decode_scale(float amax_t) {
    return amax_t > 0.0f ? __fdiv_rn(amax_t, 2688.0f) : 1.0f;
}

// Block scale from the block amax: E4M3(RNE, sat)( (amax_b / 6) * S_enc ), and the element
// multiplier r_b = S_enc / dec(s_b) (0 for a zero scale).
struct BlockScale {
    uint32_t code;
    float mult;
};
__device__ __forceinline__ BlockScale block_scale(float amax_b, float s_enc) {
    BlockScale s;
    s.code = e4m3_rne_sat(__fmul_rn(__fdiv_rn(amax_b, 6.0f), s_enc));
    s.mult = s.code ? __fdiv_rn(s_enc, e4m3_decode(s.code)) : 0.0f;
    return s;
}

// ---------------------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11).  Counter (c0, c1, c2, c3), key (k0, k1).
// ---------------------------------------------------------------------------------------
struct U4 {
    uint32_t x, y, z, w;
};

__device__ __forceinline__ U4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                            uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0, n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
        c1 = (uint32_t)p1;
        c3 = (uint32_t)p0;
        c0 = n0;
        c2 = n2;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return U4{c0, c1, c2, c3};
}

// The four 32-bit words for element group g = i/8 of stream `stream_id`.
__device__ __forceinline__ U4 sr_words(uint64_t seed, uint32_t stream_id, uint64_t g) {
    return philox4x32_10((uint32_t)g, (uint32_t)(g >> 32), stream_id, 0u, (uint32_t)seed,
                         (uint32_t)(seed >> 32));
}

// Philox with the ten round keys of one seed computed once (they depend only on the seed).
struct PhiloxKeys {
    uint32_t k0[10], k1[10];
};
__device__ __forceinline__ PhiloxKeys philox_keys(uint64_t seed) {
    PhiloxKeys k;
    uint32_t a = (uint32_t)seed, b = (uint32_t)(seed >> 32);
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        k.k0[r] = a;
        k.k1[r] = b;
        a += 0x9E3779B9u;
        b += 0xBB67AE85u;
    }
    return k;
}
__device__ __forceinline__ U4 sr_words(const PhiloxKeys& k, uint32_t stream_id, uint64_t g) {
    uint32_t c0 = (uint32_t)g, c1 = (uint32_t)(g >> 32), c2 = stream_id, c3 = 0u;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k.k0[r], n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k.k1[r];
        c1 = (uint32_t)p1;
        c3 = (uint32_t)p0;
        c0 = n0;
        c2 = n2;
    }
    return U4{c0, c1, c2, c3};
}

// ---------------------------------------------------------------------------------------
// 16-point Random Hadamard Transform: v <- 0.25 * H16 * (D v), D = diag(signs), the butterfly
// stages h = 1, 2, 4, 8 in that order, each pair (i, i+h) with bit h of i clear becoming
// (a + b, a - b).
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void rht16(float (&v)[16], uint32_t signs) {
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = ((signs >> j) & 1u) ? -v[j] : v[j];
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (i & h) continue;
            const float a = v[i], b = v[i + h];
            v[i] = __fadd_rn(a, b);
            v[i + h] = __fsub_rn(a, b);
        }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = __fmul_rn(v[j], 0.25f);
}

// The same transform on two independent 16-vectors at once (the lo and hi halves of each pair),
// with the signs already applied: each stage's adds and subtracts are f32x2 instructions.
__device__ __forceinline__ void rht16_pairs(uint64_t (&v)[16]) {
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (i & h) continue;
            const uint64_t a = v[i], b = v[i + h];
            v[i] = f2_add(a, b);
            v[i + h] = f2_sub(a, b);
        }
    }
    const uint64_t q = f2(0.25f, 0.25f);
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = f2_mul(v[j], q);
}

// A grid-stride walk over the (row, chunk) grid of a [rows][chunks_per_row] tensor without a
// division per step: the stride S = gridDim * blockDim is split once into whole rows and a
// remainder, and the position advances by carry.
struct GridWalk {
    int64_t r, k;            // current (row, chunk)
    int64_t dr, dk, cpr;     // stride in rows and chunks, chunks per row
    __device__ __forceinline__ GridWalk(int64_t start, int64_t stride, int64_t cpr_) : cpr(cpr_) {
        r = start / cpr;
        k = start - r * cpr;
        dr = stride / cpr;
        dk = stride - dr * cpr;
    }
    __device__ __forceinline__ void next() {
        r += dr;
        k += dk;
        if (k >= cpr) {
            k -= cpr;
            ++r;
        }
    }
};

// ---------------------------------------------------------------------------------------
// Position of the scale of (form row r, K-block kb) in the 128x4-tile layout read by the
// tcgen05 block-scaled MMA.
// ---------------------------------------------------------------------------------------
__host__ __device__ __forceinline__ int64_t scale_offset(int64_t r, int64_t kb, int64_t nkt) {
    return ((r >> 7) * nkt + (kb >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (kb & 3);
}

}  // namespace nvfp4
