/*
 * nvfp4_oracle.c -- plain, slow, scalar CPU oracle for the NVFP4 linear-layer hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the cpu_baseline /
 * --impl reference legs of bench.py may load this library.  The CUDA product path shares
 * no code, header, table or constant generator with it.
 *
 * Sources (the three web pages about NVIDIA's report "Pretraining Large Language Models
 * with NVFP4"; cited by page title and section):
 *   [P1] gist.science, "Pretraining Large Language Models with NVFP4", Technische
 *        Zusammenfassung: 2.A "Das NVFP4-Format" (16-element blocks, E4M3 block scales,
 *        FP32 tensor scale, about 6.25 % of a block near FP8 precision);
 *        2.B.2 "Random Hadamard Transforms" (16x16, applied only to the Wgrad inputs);
 *        2.B.3 "Zweidimensionale (2D) Block-Skalierung fuer Gewichte" (16x16 weight blocks,
 *        same quantized weight in forward and backward);
 *        2.B.4 "Stochastische Rundung" (gradients rounded stochastically, activations and
 *        weights round-to-nearest-even).
 *   [P2] webconsulting.at, "LLM-Pretraining in 4-Bit: NVIDIA stellt NVFP4-Trainingsansatz
 *        vor", "Das Wichtigste" items 1-3 (RHT, 2D scheme, stochastic rounding).
 *   [P3] brainai.pro, "NVFP4 Entraine en precision 16 bits ...", "Details techniques"
 *        (FP4 GEMMs of the fully-connected layers carry the time).
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *   - element type E2M1 {0, .5, 1, 1.5, 2, 3, 4, 6} (the pages say "FP4", MX-based);
 *   - encode scale S_enc = 6*448 / amax_t, decode scale s_t = amax_t / (6*448), both one
 *     fp32 division; amax_t == 0 gives 1 for both;
 *   - block scale s_b = E4M3_RNE_SAT( fp32(amax_b / 6) * S_enc );
 *   - element scale r_b = S_enc / dec(s_b) (0 when s_b == 0), u = v * r_b, each one fp32 op;
 *   - RNE ties go to the even code, |u| >= 6 saturates to 6, the sign is kept (-0 -> 0x8);
 *   - SR: f = (|u| - lo) / (hi - lo) (exact in fp32), round up iff r16 < ceil(f * 2^16) where
 *     r16 is a 16-bit field of Philox4x32-10 (Salmon et al., SC'11) keyed by the seed with
 *     counter (g_lo, g_hi, stream_id, 0), g = i / 8, i the element's row-major index r*K + k
 *     in the quantized form it belongs to (form row r, position k along K; for a transposed
 *     form that is source element (k, r)), field j = i mod 8 = bits [16*(j&1), +16) of
 *     output word j>>1;
 *   - RHT: one 16-sign vector per seed (bit j of word 0 of Philox(ctr=(0,0,3,0), key=seed),
 *     set = -1), v = 0.25 * H16 * (D x) with a fixed 4-stage butterfly h = 1, 2, 4, 8;
 *     transformed values stay fp32; amax_t is taken over the transformed values;
 *   - two 4-bit codes per byte, even K index in the low nibble;
 *   - scales also emitted in 128x4 tiles of 512 bytes: offset (r%32)*16 + ((r/32)%4)*4 + kb%4
 *     inside the tile of (r/128, kb/4), tiles row-tile major; padding bytes are 0.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off -fno-fast-math -pthread.
 * All fp32 arithmetic below is single IEEE binary32 operations in round-to-nearest;
 * no FMA contraction (x86-64 SSE2).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORA_OK 0
#define ORA_ERR_SHAPE 1
#define ORA_ERR_NONFINITE 2
#define ORA_ERR_ARG 3
#define ORA_ERR_NOMEM 4

/* ------------------------------------------------------------------------------------ */
/* Number formats ([P1] 2.A)                                                             */
/* ------------------------------------------------------------------------------------ */

/* Magnitudes of the eight non-negative E2M1 codes (1 sign, 2 exponent bits with bias 1,
 * 1 mantissa bit; code 1 is the subnormal 0.5). */
static const float E2M1_MAG[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

float ora_bf16_to_f32(uint16_t h) { return f32_from_bits((uint32_t)h << 16); }

/* fp32 -> bf16, round to nearest even (NaN stays NaN). */
uint16_t ora_f32_to_bf16(float f)
{
    uint32_t u = bits_from_f32(f);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

double ora_e2m1_value(uint8_t code)
{
    double m = E2M1_MAG[code & 7];
    return (code & 8) ? -m : m;
}

/* Round-to-nearest-even E2M1 encode by table search: the grid value nearest to |x|, a tie
 * going to the even code; |x| >= 6 saturates to 6; the sign bit of x is kept. */
uint8_t ora_e2m1_rne(float x)
{
    uint8_t sign = (bits_from_f32(x) >> 31) ? 8 : 0;
    double a = fabs((double)x);
    if (a >= 6.0) return sign | 7;
    int best = 0;
    double bestd = fabs(a - E2M1_MAG[0]);
    for (int c = 1; c < 8; ++c) {
        double d = fabs(a - E2M1_MAG[c]);
        if (d < bestd || (d == bestd && (c & 1) == 0)) { best = c; bestd = d; }
    }
    return sign | (uint8_t)best;
}

/* Stochastic E2M1 encode ([P1] 2.B.4): |x| lies between the grid neighbours lo <= |x| < hi;
 * f = (|x| - lo) / (hi - lo) is exact in fp32 (Sterbenz, power-of-two step); the value goes
 * up iff r16 < ceil(f * 65536).  |x| >= 6 saturates to 6.  The sign bit is kept. */
uint8_t ora_e2m1_sr(float x, uint32_t r16)
{
    uint8_t sign = (bits_from_f32(x) >> 31) ? 8 : 0;
    float a = fabsf(x);
    if (a >= 6.0f) return sign | 7;
    int c = 0;
    while (c < 7 && E2M1_MAG[c + 1] <= a) ++c;
    float lo = E2M1_MAG[c];
    float step = E2M1_MAG[c + 1] - lo;
    float f = (a - lo) / step;
    uint32_t t = (uint32_t)ceilf(f * 65536.0f);
    if (r16 < t) ++c;
    return sign | (uint8_t)c;
}

/* The SR threshold alone (ceil(f * 2^16), 0 for |x| >= 6); exposed for exhaustive checks. */
uint32_t ora_e2m1_sr_threshold(float x)
{
    float a = fabsf(x);
    if (!(a < 6.0f)) return 0;
    int c = 0;
    while (c < 7 && E2M1_MAG[c + 1] <= a) ++c;
    float lo = E2M1_MAG[c];
    float step = E2M1_MAG[c + 1] - lo;
    float f = (a - lo) / step;
    return (uint32_t)ceilf(f * 65536.0f);
}

/* Magnitude of a non-negative E4M3 ("fn" variant: no infinities, 0x7F is NaN) code. */
double ora_e4m3_value(uint8_t code)
{
    int c = code & 0x7F;
    int e = c >> 3, m = c & 7;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
    if (c == 0x7F) v = NAN;
    return (code & 0x80) ? -v : v;
}

/* Round-to-nearest-even E4M3 encode of a non-negative value, saturating at 448 (0x7E):
 * binary search of the 127-entry table of finite magnitudes, then the nearer neighbour,
 * a tie going to the even code. */
uint8_t ora_e4m3_rne_sat(float x)
{
    double a = (double)x;
    if (!(a > 0.0)) return 0;
    if (a >= 448.0) return 0x7E;
    int lo = 0, hi = 0x7E; /* invariant: value(lo) <= a < value(hi) */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (ora_e4m3_value((uint8_t)mid) <= a) lo = mid; else hi = mid;
    }
    double dl = a - ora_e4m3_value((uint8_t)lo);
    double dh = ora_e4m3_value((uint8_t)hi) - a;
    if (dl < dh) return (uint8_t)lo;
    if (dh < dl) return (uint8_t)hi;
    return (uint8_t)((lo & 1) ? hi : lo);
}

/* ------------------------------------------------------------------------------------ */
/* Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", */
/* SC'11): 10 rounds of the 4x32 S-box with multipliers 0xD2511F53 / 0xCD9E8D57 and the     */
/* Weyl key increments 0x9E3779B9 / 0xBB67AE85; the key is bumped between rounds.           */
/* ------------------------------------------------------------------------------------ */
void ora_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4])
{
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) { k0 += 0x9E3779B9u; k1 += 0xBB67AE85u; }
        uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)c0;
        uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* 16-bit random field of source element i for stochastic rounding. */
uint32_t ora_sr_bits16(uint64_t seed, uint32_t stream_id, uint64_t i)
{
    uint64_t g = i >> 3;
    uint32_t ctr[4] = {(uint32_t)g, (uint32_t)(g >> 32), stream_id, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    ora_philox4x32_10(ctr, key, out);
    unsigned f = (unsigned)(i & 7u);
    return (out[f >> 1] >> (16u * (f & 1u))) & 0xFFFFu;
}

/* ------------------------------------------------------------------------------------ */
/* Random Hadamard Transform, 16 points ([P1] 2.B.2)                                       */
/* ------------------------------------------------------------------------------------ */

/* The seeded random-sign diagonal D: bit j set means sign_j = -1. */
uint32_t ora_rht_signs(uint64_t seed)
{
    uint32_t ctr[4] = {0u, 0u, 3u, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    ora_philox4x32_10(ctr, key, out);
    return out[0] & 0xFFFFu;
}

/* v <- 0.25 * H16 * (D v): signs first, then the butterfly stages h = 1, 2, 4, 8, each pair
 * (i, i+h) with bit h of i clear becoming (a + b, a - b), then the exact scaling by 1/4. */
void ora_rht16(float v[16], uint32_t signs)
{
    for (int j = 0; j < 16; ++j)
        if ((signs >> j) & 1u) v[j] = -v[j];
    for (int h = 1; h < 16; h <<= 1) {
        for (int i = 0; i < 16; ++i) {
            if (i & h) continue;
            float a = v[i], b = v[i + h];
            v[i] = a + b;
            v[i + h] = a - b;
        }
    }
    for (int j = 0; j < 16; ++j) v[j] = v[j] * 0.25f;
}

/* ------------------------------------------------------------------------------------ */
/* Quantization of one operand form ([P1] 2.A, 2.B.2-4)                                   */
/* ------------------------------------------------------------------------------------ */

typedef struct {
    /* source: bf16 x[rows][ld], logical columns `cols` */
    const uint16_t* x;
    int64_t rows, cols, ld;
    int along;       /* 0: form rows = source rows, K = source cols; 1: form = transpose */
    int mode;        /* 0: RNE, 1: SR */
    int block;       /* 0: 1x16 along K, 1: 16x16 tiles */
    int rht;         /* 1: RHT along K of the form */
    uint64_t rht_seed, sr_seed;
    uint32_t stream_id;
    /* outputs */
    uint8_t* codes;       /* [R][K/2] */
    uint8_t* scales_rm;   /* [R][K/16] */
    uint8_t* scales_sw;   /* swizzled, ceil(R/128)*128 * ceil(K/64)*4 bytes (may be NULL) */
    uint8_t* tile_scales; /* [R/16][K/16] for 16x16 (may be NULL) */
    /* internal */
    int64_t R, K;
    float* v;             /* transformed fp32 values, [R][K] */
    float s_enc;
} ora_qjob;

static float form_value(const ora_qjob* j, int64_t r, int64_t k)
{
    int64_t sr = j->along ? k : r, sc = j->along ? r : k;
    return ora_bf16_to_f32(j->x[sr * j->ld + sc]);
}

/* index of the SR bit field of form element (r, k): its row-major position in the form */
static uint64_t form_index(const ora_qjob* j, int64_t r, int64_t k)
{
    return (uint64_t)(r * j->K + k);
}

/* swizzled offset of the scale of (form row r, K-block kb) */
int64_t ora_swizzle_offset(int64_t r, int64_t kb, int64_t K)
{
    int64_t nkt = (K / 16 + 3) / 4;
    int64_t tile = (r / 128) * nkt + kb / 4;
    return tile * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + (kb % 4);
}

int64_t ora_scales_sw_bytes(int64_t R, int64_t K)
{
    return ((R + 127) / 128) * 128 * (((K / 16) + 3) / 4) * 4;
}

static void fill_values_rows(ora_qjob* j, int64_t r0, int64_t r1)
{
    uint32_t signs = j->rht ? ora_rht_signs(j->rht_seed) : 0u;
    for (int64_t r = r0; r < r1; ++r) {
        float* row = j->v + r * j->K;
        for (int64_t k = 0; k < j->K; ++k) row[k] = form_value(j, r, k);
        if (j->rht)
            for (int64_t k = 0; k < j->K; k += 16) ora_rht16(row + k, signs);
    }
}

static uint8_t block_scale(float amax_b, float s_enc)
{
    float y = amax_b / 6.0f;
    y = y * s_enc;
    return ora_e4m3_rne_sat(y);
}

/* Encode form rows [r0, r1) (for 16x16 blocks r0 and r1 are multiples of 16). */
static void encode_rows(ora_qjob* j, int64_t r0, int64_t r1)
{
    const int64_t K = j->K, nkb = K / 16;
    for (int64_t r = r0; r < r1; ++r) {
        const float* row = j->v + r * K;
        for (int64_t kb = 0; kb < nkb; ++kb) {
            float amax_b = 0.0f;
            if (j->block == 0) {
                for (int t = 0; t < 16; ++t) amax_b = fmaxf(amax_b, fabsf(row[kb * 16 + t]));
            } else {
                int64_t rt = (r / 16) * 16;
                for (int64_t rr = rt; rr < rt + 16; ++rr)
                    for (int t = 0; t < 16; ++t)
                        amax_b = fmaxf(amax_b, fabsf(j->v[rr * K + kb * 16 + t]));
            }
            uint8_t sb = block_scale(amax_b, j->s_enc);
            float dec = (float)ora_e4m3_value(sb);
            float rb = (sb == 0) ? 0.0f : j->s_enc / dec;
            j->scales_rm[r * nkb + kb] = sb;
            if (j->scales_sw) j->scales_sw[ora_swizzle_offset(r, kb, K)] = sb;
            if (j->block == 1 && j->tile_scales && (r % 16) == 0) j->tile_scales[(r / 16) * nkb + kb] = sb;
            for (int t = 0; t < 16; t += 2) {
                uint8_t q[2];
                for (int e = 0; e < 2; ++e) {
                    int64_t k = kb * 16 + t + e;
                    float u = row[k] * rb;
                    if (j->mode == 0) q[e] = ora_e2m1_rne(u);
                    else q[e] = ora_e2m1_sr(u, ora_sr_bits16(j->sr_seed, j->stream_id, form_index(j, r, k)));
                }
                j->codes[r * (K / 2) + (kb * 16 + t) / 2] = (uint8_t)(q[0] | (q[1] << 4));
            }
        }
    }
}

typedef struct { ora_qjob* job; int64_t r0, r1; int phase; float amax; int nonfinite; } ora_slice;

static void* slice_worker(void* p)
{
    ora_slice* s = (ora_slice*)p;
    if (s->phase == 0) {
        fill_values_rows(s->job, s->r0, s->r1);
        float m = 0.0f;
        int nf = 0;
        for (int64_t r = s->r0; r < s->r1; ++r)
            for (int64_t k = 0; k < s->job->K; ++k) {
                float a = fabsf(s->job->v[r * s->job->K + k]);
                if (!isfinite(a)) nf = 1; else m = fmaxf(m, a);
            }
        s->amax = m;
        s->nonfinite = nf;
    } else {
        encode_rows(s->job, s->r0, s->r1);
    }
    return NULL;
}

static int run_slices(ora_qjob* job, int phase, int nthreads, float* amax, int* nonfinite)
{
    int64_t gran = (job->block == 1) ? 16 : 1;
    int64_t units = (job->R + gran - 1) / gran;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > units) nthreads = (int)(units > 0 ? units : 1);
    ora_slice* sl = (ora_slice*)calloc((size_t)nthreads, sizeof(ora_slice));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!sl || !th) { free(sl); free(th); return ORA_ERR_NOMEM; }
    for (int t = 0; t < nthreads; ++t) {
        sl[t].job = job;
        sl[t].phase = phase;
        sl[t].r0 = (units * t / nthreads) * gran;
        sl[t].r1 = (units * (t + 1) / nthreads) * gran;
        if (sl[t].r1 > job->R) sl[t].r1 = job->R;
    }
    if (nthreads == 1) slice_worker(&sl[0]);
    else {
        for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, slice_worker, &sl[t]);
        for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    }
    if (phase == 0) {
        float m = 0.0f;
        int nf = 0;
        for (int t = 0; t < nthreads; ++t) { m = fmaxf(m, sl[t].amax); nf |= sl[t].nonfinite; }
        *amax = m;
        *nonfinite = nf;
    }
    free(sl);
    free(th);
    return ORA_OK;
}

/*
 * Quantize one operand form.  Returns ORA_OK, ORA_ERR_SHAPE (K % 16, or R % 16 for 16x16),
 * ORA_ERR_ARG, ORA_ERR_NONFINITE (NaN/Inf among the transformed values; outputs undefined)
 * or ORA_ERR_NOMEM.  amax_out receives amax_t, s_t_out the decode tensor scale.
 * `nthreads` splits the form rows into contiguous slices (bit-identical for any count).
 */
int ora_quantize(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, int along, int mode,
                 int block, int rht, uint64_t rht_seed, uint64_t sr_seed, uint32_t stream_id,
                 uint8_t* codes, uint8_t* scales_rm, uint8_t* scales_sw, uint8_t* tile_scales,
                 float* amax_out, float* s_t_out, int nthreads)
{
    ora_qjob j;
    memset(&j, 0, sizeof(j));
    if (rows < 0 || cols < 0 || ld < cols || (mode != 0 && mode != 1) || (block != 0 && block != 1)) return ORA_ERR_ARG;
    j.x = x; j.rows = rows; j.cols = cols; j.ld = ld; j.along = along; j.mode = mode; j.block = block;
    j.rht = rht; j.rht_seed = rht_seed; j.sr_seed = sr_seed; j.stream_id = stream_id;
    j.codes = codes; j.scales_rm = scales_rm; j.scales_sw = scales_sw; j.tile_scales = tile_scales;
    j.R = along ? cols : rows;
    j.K = along ? rows : cols;
    if (j.K % 16 != 0) return ORA_ERR_SHAPE;
    if (block == 1 && j.R % 16 != 0) return ORA_ERR_SHAPE;
    if (scales_sw) memset(scales_sw, 0, (size_t)ora_scales_sw_bytes(j.R, j.K));
    if (j.R == 0 || j.K == 0) { *amax_out = 0.0f; *s_t_out = 1.0f; return ORA_OK; }
    j.v = (float*)malloc((size_t)(j.R * j.K) * sizeof(float));
    if (!j.v) return ORA_ERR_NOMEM;
    float amax = 0.0f;
    int nonfinite = 0;
    int st = run_slices(&j, 0, nthreads, &amax, &nonfinite);
    if (st == ORA_OK && nonfinite) st = ORA_ERR_NONFINITE;
    if (st == ORA_OK) {
        /* tensor scales ([P1] 2.A, two-level scaling) */
        float s_enc = 1.0f, s_t = 1.0f;
        if (amax > 0.0f) {
            s_enc = 2688.0f / amax;
            s_t = amax / 2688.0f;
        }
        j.s_enc = s_enc;
        *amax_out = amax;
        *s_t_out = s_t;
        st = run_slices(&j, 1, nthreads, NULL, NULL);
    }
    free(j.v);
    return st;
}

/*
 * 2D-scaled weight in transposed layout without requantizing ([P1] 2.B.3): codes_t[k][r] is
 * the code of (r, k); the tile grid is transposed; scales of the transposed form follow.
 * Input: codes [R][K/2], tile_scales [R/16][K/16].  Output: codes_t [K][R/2], scales_rm_t
 * [K][R/16], scales_sw_t (swizzled for a K x R form), tile_scales_t [K/16][R/16].
 */
int ora_transpose_2d(const uint8_t* codes, const uint8_t* tile_scales, int64_t R, int64_t K,
                     uint8_t* codes_t, uint8_t* scales_rm_t, uint8_t* scales_sw_t, uint8_t* tile_scales_t)
{
    if (R % 16 || K % 16) return ORA_ERR_SHAPE;
    if (scales_sw_t) memset(scales_sw_t, 0, (size_t)ora_scales_sw_bytes(K, R));
    memset(codes_t, 0, (size_t)(K * (R / 2)));
    for (int64_t r = 0; r < R; ++r)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = codes[r * (K / 2) + k / 2];
            uint8_t q = (k & 1) ? (byte >> 4) : (byte & 15);
            codes_t[k * (R / 2) + r / 2] |= (uint8_t)((r & 1) ? (q << 4) : q);
        }
    for (int64_t a = 0; a < R / 16; ++a)
        for (int64_t b = 0; b < K / 16; ++b) {
            uint8_t s = tile_scales[a * (K / 16) + b];
            if (tile_scales_t) tile_scales_t[b * (R / 16) + a] = s;
            for (int64_t kk = b * 16; kk < b * 16 + 16; ++kk) {
                scales_rm_t[kk * (R / 16) + a] = s;
                if (scales_sw_t) scales_sw_t[ora_swizzle_offset(kk, a, R)] = s;
            }
        }
    return ORA_OK;
}

/* Dequantize a form: out[r][k] = e2m1(code) * e4m3(s_b) * s_t, exact in fp64. */
void ora_dequantize(const uint8_t* codes, const uint8_t* scales_rm, float s_t, int64_t R, int64_t K, double* out)
{
    for (int64_t r = 0; r < R; ++r)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = codes[r * (K / 2) + k / 2];
            uint8_t q = (k & 1) ? (byte >> 4) : (byte & 15);
            out[r * K + k] = ora_e2m1_value(q) * ora_e4m3_value(scales_rm[r * (K / 16) + k / 16]) * (double)s_t;
        }
}

/* ------------------------------------------------------------------------------------ */
/* Block-scaled GEMM reference ([P3] Details techniques; [P1] 3): D[i][j] = sum_k a_ik b_jk  */
/* over the dequantized operands, in fp64.  Also returns sum_k |a_ik b_jk| for tolerances.  */
/* ------------------------------------------------------------------------------------ */

/* Decode tables filled from the scalar decoders above before any worker thread starts. */
static double E2M1_TAB[16];
static double E4M3_TAB[256];

static void init_decode_tables(void)
{
    for (int c = 0; c < 16; ++c) E2M1_TAB[c] = ora_e2m1_value((uint8_t)c);
    for (int c = 0; c < 256; ++c) E4M3_TAB[c] = ora_e4m3_value((uint8_t)c);
}

static double deq(const uint8_t* codes, const uint8_t* scales_rm, double s_t, int64_t K, int64_t r, int64_t k)
{
    uint8_t byte = codes[r * (K / 2) + k / 2];
    uint8_t q = (k & 1) ? (byte >> 4) : (byte & 15);
    return E2M1_TAB[q] * E4M3_TAB[scales_rm[r * (K / 16) + k / 16]] * s_t;
}

typedef struct {
    const uint8_t *ac, *as, *bc, *bs;
    double ast, bst;
    int64_t K;
    const int64_t *ii, *jj;
    int64_t n0, n1;
    double *d, *sabs;
} ora_gjob;

static void* gemm_worker(void* p)
{
    ora_gjob* g = (ora_gjob*)p;
    for (int64_t t = g->n0; t < g->n1; ++t) {
        double acc = 0.0, sa = 0.0;
        for (int64_t k = 0; k < g->K; ++k) {
            double prod = deq(g->ac, g->as, g->ast, g->K, g->ii[t], k) * deq(g->bc, g->bs, g->bst, g->K, g->jj[t], k);
            acc += prod;
            sa += fabs(prod);
        }
        g->d[t] = acc;
        if (g->sabs) g->sabs[t] = sa;
    }
    return NULL;
}

/* Sampled outputs (ii[t], jj[t]) of D = A * B^T over K for quantized forms A [M][K], B [N][K]. */
int ora_gemm_sampled(const uint8_t* a_codes, const uint8_t* a_scales_rm, float a_st,
                     const uint8_t* b_codes, const uint8_t* b_scales_rm, float b_st, int64_t K,
                     const int64_t* ii, const int64_t* jj, int64_t n, double* d_out, double* sabs_out,
                     int nthreads)
{
    if (K % 16) return ORA_ERR_SHAPE;
    init_decode_tables();
    if (nthreads < 1) nthreads = 1;
    if (nthreads > n) nthreads = (int)(n > 0 ? n : 1);
    ora_gjob* gj = (ora_gjob*)calloc((size_t)nthreads, sizeof(ora_gjob));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!gj || !th) { free(gj); free(th); return ORA_ERR_NOMEM; }
    for (int t = 0; t < nthreads; ++t) {
        gj[t] = (ora_gjob){a_codes, a_scales_rm, b_codes, b_scales_rm, (double)a_st, (double)b_st, K,
                           ii, jj, n * t / nthreads, n * (t + 1) / nthreads, d_out, sabs_out};
    }
    if (nthreads == 1) gemm_worker(&gj[0]);
    else {
        for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, gemm_worker, &gj[t]);
        for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    }
    free(gj);
    free(th);
    return ORA_OK;
}

/* Full D = A * B^T (small sizes): dequantize both operands, then a plain triple loop. */
int ora_gemm_full(const uint8_t* a_codes, const uint8_t* a_scales_rm, float a_st,
                  const uint8_t* b_codes, const uint8_t* b_scales_rm, float b_st,
                  int64_t M, int64_t N, int64_t K, double* d_out, double* sabs_out)
{
    if (K % 16) return ORA_ERR_SHAPE;
    double* a = (double*)malloc((size_t)(M * K) * sizeof(double));
    double* b = (double*)malloc((size_t)(N * K) * sizeof(double));
    if (!a || !b) { free(a); free(b); return ORA_ERR_NOMEM; }
    ora_dequantize(a_codes, a_scales_rm, a_st, M, K, a);
    ora_dequantize(b_codes, b_scales_rm, b_st, N, K, b);
    for (int64_t i = 0; i < M; ++i)
        for (int64_t jn = 0; jn < N; ++jn) {
            double acc = 0.0, sa = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double prod = a[i * K + k] * b[jn * K + k];
                acc += prod;
                sa += fabs(prod);
            }
            d_out[i * N + jn] = acc;
            if (sabs_out) sabs_out[i * N + jn] = sa;
        }
    free(a);
    free(b);
    return ORA_OK;
}

/* ------------------------------------------------------------------------------------ */
/* GeLU glue of the one-FFN training step (not part of the pages' method): exact (erf)     */
/* form g = x * Phi(x), evaluated in fp64 and rounded to bf16.  Phi(x) = erfc(-x/sqrt 2)/2:  */
/* the same function as (1 + erf(x/sqrt 2))/2 without its cancellation for negative x.     */
/* ------------------------------------------------------------------------------------ */
void ora_gelu_fwd(const uint16_t* h, int64_t n, uint16_t* g)
{
    for (int64_t i = 0; i < n; ++i) {
        double x = ora_bf16_to_f32(h[i]);
        double y = 0.5 * x * erfc(-x / sqrt(2.0));
        g[i] = ora_f32_to_bf16((float)y);
    }
}

/* dH = dG * GeLU'(H), GeLU'(x) = Phi(x) + x * phi(x). */
void ora_gelu_bwd(const uint16_t* h, const uint16_t* dg, int64_t n, uint16_t* dh)
{
    const double inv_sqrt_2pi = 0.39894228040143267794;
    for (int64_t i = 0; i < n; ++i) {
        double x = ora_bf16_to_f32(h[i]);
        double d = ora_bf16_to_f32(dg[i]);
        double cdf = 0.5 * erfc(-x / sqrt(2.0));
        double pdf = inv_sqrt_2pi * exp(-0.5 * x * x);
        dh[i] = ora_f32_to_bf16((float)(d * (cdf + x * pdf)));
    }
}

/* ------------------------------------------------------------------------------------ */
/* Batch helpers for exhaustive / statistical pins                                        */
/* ------------------------------------------------------------------------------------ */
void ora_e2m1_rne_batch(const float* x, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = ora_e2m1_rne(x[i]);
}

void ora_e2m1_sr_batch(const float* x, const uint32_t* r16, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = ora_e2m1_sr(x[i], r16[i]);
}

void ora_e2m1_sr_threshold_batch(const float* x, int64_t n, uint32_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = ora_e2m1_sr_threshold(x[i]);
}

void ora_e4m3_rne_sat_batch(const float* x, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = ora_e4m3_rne_sat(x[i]);
}

void ora_sr_bits16_batch(uint64_t seed, uint32_t stream_id, const uint64_t* idx, int64_t n, uint32_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = ora_sr_bits16(seed, stream_id, idx[i]);
}

/* Philox blocks for counters (c_lo + t, c_hi, stream, 0), t = 0..n-1. */
void ora_philox_batch(uint64_t seed, uint32_t stream_id, uint64_t g0, int64_t n, uint32_t* out4)
{
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    for (int64_t t = 0; t < n; ++t) {
        uint64_t g = g0 + (uint64_t)t;
        uint32_t ctr[4] = {(uint32_t)g, (uint32_t)(g >> 32), stream_id, 0u};
        ora_philox4x32_10(ctr, key, out4 + 4 * t);
    }
}

/* ------------------------------------------------------------------------------------ */
/* MXFP4, the pages' comparison format (gist.science 2.A: blocks of 32 elements, UE8M0    */
/* scale factors, no tensor scale).  The pages give no rule for the scale; the reading    */
/* taken is the microscaling one: the block's shared exponent is floor(log2 amax_b) - 2   */
/* (2 = the largest E2M1 exponent, 6 = 1.5 * 2^2), stored as the UE8M0 code E + 127,      */
/* clamped to [0, 254] (255 is NaN); an all-zero block gets code 0.  Elements are         */
/* u = v / 2^E (exact: a power of two), encoded to E2M1 by RNE or SR exactly as NVFP4's,   */
/* saturating to 6.  SR fields are indexed by the element's row-major position.           */
/* ------------------------------------------------------------------------------------ */
uint8_t ora_ue8m0_of_amax(float amax)
{
    if (!(amax > 0.0f)) return 0;
    int e2;
    (void)frexpf(amax, &e2);          /* amax = m * 2^e2, m in [0.5, 1): floor(log2 amax) = e2 - 1 */
    int code = (e2 - 1) - 2 + 127;
    if (code < 0) code = 0;
    if (code > 254) code = 254;
    return (uint8_t)code;
}

/* x [rows][cols] bf16 (leading dimension ld), cols % 32 == 0 -> codes [rows][cols/2] (even k in
   the low nibble), scales [rows][cols/32] UE8M0. */
int ora_quantize_mx(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, int mode, uint64_t sr_seed,
                    uint32_t stream_id, uint8_t* codes, uint8_t* scales)
{
    if (rows < 0 || cols < 0 || cols % 32 != 0 || ld < cols) return ORA_ERR_SHAPE;
    if (mode != 0 && mode != 1) return ORA_ERR_ARG;
    const int64_t nb = cols / 32;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            float amax = 0.0f;
            for (int t = 0; t < 32; ++t) {
                float v = ora_bf16_to_f32(x[r * ld + b * 32 + t]);
                if (isnan(v) || isinf(v)) return ORA_ERR_NONFINITE;
                amax = fmaxf(amax, fabsf(v));
            }
            const uint8_t sc = ora_ue8m0_of_amax(amax);
            scales[r * nb + b] = sc;
            const int e = (int)sc - 127;
            for (int t = 0; t < 32; t += 2) {
                uint8_t q[2];
                for (int j = 0; j < 2; ++j) {
                    const int64_t k = b * 32 + t + j;
                    const float u = ldexpf(ora_bf16_to_f32(x[r * ld + k]), -e);
                    q[j] = mode == 0 ? ora_e2m1_rne(u)
                                     : ora_e2m1_sr(u, ora_sr_bits16(sr_seed, stream_id, (uint64_t)(r * cols + k)));
                }
                codes[r * (cols / 2) + (b * 32 + t) / 2] = (uint8_t)(q[0] | (q[1] << 4));
            }
        }
    }
    return ORA_OK;
}

/* MXFP4 dequantize: value = E2M1(code) * 2^(scale - 127), exact in fp64 (codes [R][K/2] with the
   even element in the low nibble, UE8M0 scales [R][K/32] row-major; scale 255 is NaN and never
   produced by ora_quantize_mx). */
void ora_dequantize_mx(const uint8_t* codes, const uint8_t* scales, int64_t R, int64_t K, double* out)
{
    for (int64_t r = 0; r < R; ++r)
        for (int64_t k = 0; k < K; ++k) {
            const uint8_t byte = codes[r * (K / 2) + k / 2];
            const uint8_t nib = (k & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15u);
            const double scale = ldexp(1.0, (int)scales[r * (K / 32) + k / 32] - 127);
            out[r * K + k] = ora_e2m1_value(nib) * scale;
        }
}

/* The MXFP4 scales [R][K/32] in the 128x4 tiles the block-scaled MMA reads: entry (r, kb) at
   ((r/128)*ceil(K/128) + kb/4)*512 + (r%32)*16 + ((r/32)%4)*4 + kb%4, padding 0 (sw holds
   ceil(R/128)*128 * ceil(K/128)*4 bytes). */
void ora_mx_scales_swizzle(const uint8_t* scales, int64_t R, int64_t K, uint8_t* sw)
{
    const int64_t nkt = (K / 32 + 3) / 4;
    memset(sw, 0, (size_t)(((R + 127) / 128) * 128 * nkt * 4));
    for (int64_t r = 0; r < R; ++r)
        for (int64_t kb = 0; kb < K / 32; ++kb)
            sw[((r / 128) * nkt + kb / 4) * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + (kb % 4)] = scales[r * (K / 32) + kb];
}
