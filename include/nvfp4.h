/*
 * nvfp4.h -- C ABI of libnvfp4: NVFP4 quantization fused into block-scaled FP4 GEMMs for the
 * fprop, dgrad and wgrad GEMMs of a linear layer, on one B200 (sm_100a).
 *
 * What the operations are follows the pages on NVIDIA's report "Pretraining Large Language
 * Models with NVFP4" (gist.science, Technische Zusammenfassung 2.A and 2.B; webconsulting.at,
 * "Das Wichtigste"; brainai.pro, "Details techniques"):
 *   - NVFP4 = 4-bit E2M1 elements, one E4M3 scale per 16 consecutive elements, one FP32 scale
 *     per tensor (2.A "Das NVFP4-Format");
 *   - weights use 16x16 2D blocks so forward and backward see the same quantized weight
 *     (2.B.3);
 *   - a seeded 16-point Random Hadamard Transform is applied along K to both Wgrad operands
 *     only (2.B.2);
 *   - gradients are rounded stochastically, activations and weights round-to-nearest-even
 *     (2.B.4);
 *   - the GEMMs run on the Blackwell FP4 tensor cores (3, "Hardware-Nutzung").
 *
 * Conventions for every call:
 *   - All tensor pointers are caller-owned DEVICE pointers.  The library never allocates,
 *     never frees, never prints and never throws across this boundary.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream)
 *     and returns after validating its arguments and enqueuing its kernels.  Argument checks
 *     are synchronous and happen before any launch: a non-OK status means nothing was enqueued
 *     (except NVFP4_ERR_CUDA, which reports a failed launch; the CUDA error is consumed).
 *   - Conditions detected on the device (NaN/Inf input, a device-side wait that ran out of its
 *     time budget) set flags in the caller's workspace; read them with nvfp4_poll().
 *   - Layouts: bf16 inputs are row-major with a leading dimension in elements.  A quantized
 *     form (nvfp4_tensor) has `rows` rows and `k` elements along the GEMM reduction axis:
 *       codes        [rows][k/2] bytes, K-major, element 2j in the low nibble of byte j;
 *       scales       E4M3 block scales in 128x4 tiles of 512 bytes: the scale of (row r,
 *                    block kb = k_index/16) sits at ((r/128)*ceil(k/64) + kb/4)*512
 *                    + (r%32)*16 + ((r/32)%4)*4 + kb%4; padding bytes are zero (this is the
 *                    layout the tcgen05 block-scaled MMA reads through tcgen05.cp);
 *       tile_scales  16x16 forms only: compact grid [rows/16][k/16] (may be NULL);
 *       tensor_scale one fp32: the decode scale s_t = amax_t / (6*448).
 *     A value is reconstructed as e2m1(code) * e4m3(scale) * s_t.
 *   - Alignment: every device pointer 16-byte aligned.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so the header needs no CUDA include. */
typedef struct CUstream_st* nvfp4_stream_t;

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_NULL = 1,        /* a required pointer is NULL */
    NVFP4_ERR_ALIGN = 2,       /* a pointer or leading dimension breaks the 16-byte rule */
    NVFP4_ERR_SHAPE = 3,       /* a size violates the operation's shape rule (see each call) */
    NVFP4_ERR_ARG = 4,         /* an enum or flag out of range, or inconsistent operands */
    NVFP4_ERR_WORKSPACE = 5,   /* workspace NULL */
    NVFP4_ERR_CUDA = 6,        /* a CUDA launch or runtime call failed */
    NVFP4_ERR_NONFINITE = 7,   /* (nvfp4_poll) NaN or Inf seen by an amax pass */
    NVFP4_ERR_TIMEOUT = 8,     /* (nvfp4_poll) a device-side wait ran out of its time budget */
    NVFP4_ERR_UNSUPPORTED = 9, /* the device is not sm_100 */
    NVFP4_ERR_LIMIT = 10       /* a size exceeds a fixed limit of the call */
} nvfp4_status;

typedef enum { NVFP4_RNE = 0, NVFP4_SR = 1 } nvfp4_round;
typedef enum { NVFP4_BLOCK_1x16 = 0, NVFP4_BLOCK_16x16 = 1 } nvfp4_block;
typedef enum { NVFP4_OUT_BF16 = 0, NVFP4_OUT_FP32 = 1 } nvfp4_dtype;

/* Philox stream ids used by the linear layer (the counter's third word). */
#define NVFP4_STREAM_DGRAD 1u   /* dY, 1x16 along the output features (dgrad operand) */
#define NVFP4_STREAM_WGRAD 2u   /* dY^T after the RHT, 1x16 along tokens (wgrad operand) */
#define NVFP4_STREAM_RHT 3u     /* reserved: the RHT sign draw */

typedef struct {
    uint8_t* codes;
    uint8_t* scales;
    uint8_t* tile_scales;
    float* tensor_scale;
    int64_t rows;
    int64_t k;
    int32_t block;     /* nvfp4_block */
    int32_t reserved;
} nvfp4_tensor;

/* ---- sizes (host, pure functions) ------------------------------------------------------ */
size_t nvfp4_codes_bytes(int64_t rows, int64_t k);       /* rows * k / 2 */
size_t nvfp4_scales_bytes(int64_t rows, int64_t k);      /* ceil(rows/128)*128 * ceil(k/64)*4 */
size_t nvfp4_tile_scales_bytes(int64_t rows, int64_t k); /* (rows/16) * (k/16) */
size_t nvfp4_workspace_bytes(void);                      /* 256 */

/* Zero a workspace (flags and amax slots).  Call once after allocating it. */
nvfp4_status nvfp4_workspace_init(void* ws, nvfp4_stream_t stream);

/*
 * Quantize one operand form of a bf16 tensor x[rows][ldx] (logical width `cols`).
 * along = 0: the form is x itself (form rows = rows, k = cols).
 * along = 1: the form is x^T (form rows = cols, k = rows) -- the token-major wgrad operands.
 * block: 1x16 along k, or 16x16 tiles (weights).  rht = 1 applies the seeded 16-point RHT
 * along k before anything else (1x16 only).  mode = NVFP4_SR draws one 16-bit Philox field
 * per element: key = sr_seed, counter = (i/8 lo, i/8 hi, stream_id, 0), field i mod 8, where
 * i = the element's row-major index in the form (form row * k + position along k: r*cols + c
 * for along = 0, c*rows + r for along = 1).  The RHT signs are bit j of word 0 of
 * Philox(key = rht_seed, counter = (0, 0, 3, 0)), set = -1.
 * Two passes over x: an amax reduction (over the transformed values when rht = 1) and the
 * quantize pass; tensor scales S_enc = 2688/amax_t, s_t = amax_t/2688 (1 and 1 if amax_t == 0).
 * Shape rules: k % 16 == 0; along = 1 or 16x16 needs form rows % 16 == 0 and k % 16 == 0;
 * cols % 16 == 0 always.  rows or cols == 0 is a no-op that writes s_t = 1.
 * out: codes/scales/tensor_scale required, tile_scales required for 16x16 (else ignored);
 * out->rows/k/block are written by the call.  ws: a workspace of nvfp4_workspace_bytes().
 */
nvfp4_status nvfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ldx, int along,
                            nvfp4_round mode, nvfp4_block block, int rht, uint64_t rht_seed,
                            uint64_t sr_seed, uint32_t stream_id, nvfp4_tensor* out, void* ws,
                            nvfp4_stream_t stream);

/*
 * One read of x, two forms (gist.science 2.B.2: RHT only for the Wgrad inputs):
 *   out_row: along = 0, 1x16, no RHT, rounding `mode`, Philox stream `stream_row`
 *            (fprop operand X, dgrad operand dY);
 *   out_col: along = 1, 1x16, RHT (rht_seed), rounding `mode`, Philox stream `stream_col`
 *            (wgrad operands X^T, dY^T).
 * Results are bit-identical to two nvfp4_quantize calls with the same arguments.
 * Shape rules: rows % 16 == 0, cols % 16 == 0.
 */
nvfp4_status nvfp4_quantize_dual(const void* x, int64_t rows, int64_t cols, int64_t ldx,
                                 nvfp4_round mode, uint64_t rht_seed, uint64_t sr_seed,
                                 uint32_t stream_row, uint32_t stream_col, nvfp4_tensor* out_row,
                                 nvfp4_tensor* out_col, void* ws, nvfp4_stream_t stream);

/*
 * Data-parallel token shards.  The tensor scale comes from the amax of the whole tensor
 * (gist.science 2.A), so ranks that each hold a shard of the tokens split the two passes and
 * reduce the amax between them:
 *   1. nvfp4_amax(shard, rht = 1, rht_seed, ws): the shard's plain amax and the amax after the
 *      16-point RHT along rows, written as two uint32 fp32 bit patterns at byte offset
 *      nvfp4_workspace_amax_offset() of ws (reset first).  rows % 16 == 0 when rht = 1.
 *   2. the caller reduces both words with MAX across ranks (for non-negative floats the bit
 *      patterns order like the values, so an integer MAX over int32 is exact);
 *   3. nvfp4_quantize_dual_shard(shard, ..., row_offset, rows_total, ...): pass 2 of
 *      nvfp4_quantize_dual with the tensor scales of those reduced amaxes.  The shard holds rows
 *      [row_offset, row_offset + rows) of a rows_total-row tensor, and SR fields are indexed in
 *      that tensor's forms (row form: (row_offset + r) * cols + c; column form:
 *      c * rows_total + row_offset + r).
 * Each shard's forms then equal, bit for bit, its rows (row form) and its K range (column form)
 * of nvfp4_quantize_dual over the whole tensor.  Shape rules: those of nvfp4_quantize_dual, and
 * row_offset % 16 == 0, row_offset + rows <= rows_total.  The shard's column form has k = rows.
 */
nvfp4_status nvfp4_amax(const void* x, int64_t rows, int64_t cols, int64_t ldx, int rht,
                        uint64_t rht_seed, void* ws, nvfp4_stream_t stream);
size_t nvfp4_workspace_amax_offset(void);
nvfp4_status nvfp4_quantize_dual_shard(const void* x, int64_t rows, int64_t cols, int64_t ldx,
                                       int64_t row_offset, int64_t rows_total, nvfp4_round mode,
                                       uint64_t rht_seed, uint64_t sr_seed, uint32_t stream_row,
                                       uint32_t stream_col, nvfp4_tensor* out_row,
                                       nvfp4_tensor* out_col, void* ws, nvfp4_stream_t stream);

/*
 * 16x16 weight quantization (gist.science 2.B.3), RNE, writing the forward form w_q
 * ([rows][cols], k = cols) and, if w_qt is not NULL, the transposed dgrad form
 * ([cols][rows], k = rows) from the same registers -- bit-identical to nvfp4_transpose_2d of
 * w_q.  Shape rules: rows % 16 == 0, cols % 16 == 0.  tile_scales of w_q is required.
 */
nvfp4_status nvfp4_quantize_weight(const void* w, int64_t rows, int64_t cols, int64_t ldw,
                                   nvfp4_tensor* w_q, nvfp4_tensor* w_qt, void* ws,
                                   nvfp4_stream_t stream);

/*
 * Transposed layout of a 16x16-quantized tensor without requantizing (gist.science 2.B.3):
 * wt->codes[k][r] = w->codes[r][k], tile grid transposed, same tensor scale (copied).
 * w->block must be NVFP4_BLOCK_16x16 with tile_scales; wt->tile_scales may be NULL.
 */
nvfp4_status nvfp4_transpose_2d(const nvfp4_tensor* w, nvfp4_tensor* wt, nvfp4_stream_t stream);

/*
 * D[M][N] = s_tA * s_tB * sum_k A[m][k] * B[n][k]: both operands K-major quantized forms with
 * the same k (brainai.pro "Details techniques": the FP4 GEMMs of the fully connected layers).
 * M = a->rows, N = b->rows, K = a->k.  fp32 accumulation in tensor memory; bf16 or fp32 output
 * with leading dimension ldd (elements).  Shape rules: K % 32 == 0 and K > 0; M, N >= 1;
 * ldd >= N and ldd * sizeof(out) % 16 == 0.  ws receives the timeout flag.  For M >= 256 the
 * call runs the SM-pair kernel (a cluster of two CTAs per 256 x 256 output tile); the environment
 * variable NVFP4_GEMM_VARIANT=1sm, read on every call, selects the 1-SM kernel for every shape.
 */
nvfp4_status nvfp4_gemm(const nvfp4_tensor* a, const nvfp4_tensor* b, void* d, int64_t ldd,
                        nvfp4_dtype out_dtype, void* ws, nvfp4_stream_t stream);

/*
 * The same product as nvfp4_gemm with fp32 output, ADDED into row shards instead of stored: the
 * data-parallel weight gradient (gist.science 2.B: dW is a sum over tokens, so each replica holds a
 * K-partial that the replicas sum), reduced as the GEMM's epilogue writes it.  Owner o receives
 * rows [o * owner_rows, min(M, (o + 1) * owner_rows)) of D: shards[o][r][c] += D[o * owner_rows + r][c],
 * row stride ldd (elements).  shards is a HOST array of n_owners device addresses valid on the
 * calling device (local buffers, or other GPUs' buffers through peer mappings); each output tile
 * is added by the TMA engine (an fp32 bulk tensor reduce-add) once, so a shard accumulates whatever
 * it held before: zero it for a plain reduce-scatter, or pass one owner (owner_rows >= M) to
 * accumulate a gradient into an existing fp32 buffer.  Every add of the call is complete in memory
 * when the call's work on `stream` is complete; the caller orders the shards' later readers (a
 * stream event, or a collective as a barrier between GPUs).  Adds from several calls into one
 * shard at the same time are per-element reductions in an order that is not fixed, so their sum
 * is reproducible only up to fp32 rounding order.  Shape rules: those of nvfp4_gemm;
 * 1 <= n_owners <= 8; owner_rows % 32 == 0 and n_owners == ceil(M / owner_rows); shards 16-byte
 * aligned; ldd * 4 % 16 == 0 (NVFP4_ERR_SHAPE / NVFP4_ERR_ALIGN / NVFP4_ERR_NULL otherwise,
 * before any device work).
 */
nvfp4_status nvfp4_gemm_reduce_scatter(const nvfp4_tensor* a, const nvfp4_tensor* b, float* const* shards,
                                       int n_owners, int64_t owner_rows, int64_t ldd, void* ws,
                                       nvfp4_stream_t stream);

/*
 * nvfp4_gemm with bf16 output that also produces the output's amax for the quantize call that
 * will read it (gist.science 2.A: the FP32 tensor scale comes from the amax of the whole tensor,
 * a pass over it that the producer can take over): the plain amax of the stored bf16 D and the
 * amax of its 16-point RHT along the rows (signs from rht_seed, the transform of the wgrad form
 * of D as a token-major operand) are written into amax_ws's amax words, exactly as nvfp4_amax(D,
 * rht = 1, rht_seed) would: the same fp32 operations on the same bf16 values.  A linear context
 * whose workspace is amax_ws can then quantize D with amax_ready set, and
 * nvfp4_quantize_dual_shard(D, 0, rows, ...) with amax_ws uses the words as they are.  amax_ws's
 * words are reset first; a non-finite output raises the non-finite flag in ws.  Shape rules: those
 * of nvfp4_gemm, and M % 16 == 0.
 */
nvfp4_status nvfp4_gemm_amax(const nvfp4_tensor* a, const nvfp4_tensor* b, void* d, int64_t ldd,
                             uint64_t rht_seed, void* amax_ws, void* ws, nvfp4_stream_t stream);

/*
 * Linear layer y = x w^T with NVFP4 GEMMs (gist.science 2.B): all buffers caller-owned.
 *   xq      [T][d]   1x16 RNE           (fprop A)
 *   xq_rht  [d][T]   RHT 1x16 RNE       (wgrad B)
 *   wq      [n][d]   16x16 RNE          (fprop B; tile_scales required)
 *   wqt     [d][n]   16x16 transposed   (dgrad B)
 *   dyq     [T][n]   1x16 SR stream 1   (dgrad A)
 *   dyq_rht [n][T]   RHT 1x16 SR stream 2 (wgrad A)
 * w_cached != 0 makes nvfp4_linear_fwd reuse wq/wqt as they are.  Shape rules: T % 64 == 0,
 * d % 64 == 0, n % 64 == 0 (each is a K of one GEMM and a 16-row tile dimension).
 */
typedef struct {
    int64_t T, d, n;
    uint64_t rht_seed;
    nvfp4_tensor xq, xq_rht, wq, wqt, dyq, dyq_rht;
    void* ws;
    int32_t w_cached;
    /* nonzero: the amax words of the next call's input (x for nvfp4_linear_fwd, dy for
     * nvfp4_linear_bwd) are already in ws, written by a producer that fused them
     * (nvfp4_gelu_fwd_amax, nvfp4_gelu_bwd_amax, or nvfp4_amax + a reduction); the call then
     * skips its amax pass and sets the field back to 0 */
    int32_t amax_ready;
    /* optional: the amax words of this layer's outputs for the contexts that will quantize them.
     * Non-null y_amax_ws makes nvfp4_linear_fwd's fprop GEMM also write y's plain amax and its RHT
     * amax (signs from y_rht_seed) into that workspace (nvfp4_gemm_amax; T % 16 == 0 holds); the
     * consuming context (y is its x) then sets amax_ready.  dx_amax_ws / dx_rht_seed do the same
     * for dx in nvfp4_linear_bwd (dx is the consuming context's dy).  Null: off. */
    void* y_amax_ws;
    uint64_t y_rht_seed;
    void* dx_amax_ws;
    uint64_t dx_rht_seed;
} nvfp4_linear_ctx;

/* Forward: quantize X (both forms), quantize W (16x16, both layouts) unless cached, then
 * y[T][n] (bf16) = GEMM(xq, wq). */
nvfp4_status nvfp4_linear_fwd(const void* x, const void* w, void* y, nvfp4_linear_ctx* ctx,
                              nvfp4_stream_t stream);

/* Backward: quantize dY (both forms, SR with sr_seed), dx[T][d] (bf16) = GEMM(dyq, wqt),
 * dw[n][d] (fp32) = GEMM(dyq_rht, xq_rht).  dx or dw may be NULL to skip that GEMM. */
nvfp4_status nvfp4_linear_bwd(const void* dy, uint64_t sr_seed, void* dx, float* dw,
                              nvfp4_linear_ctx* ctx, nvfp4_stream_t stream);

/* GeLU glue of the one-FFN training step (exact erf form, fp32 math, bf16 in and out; the pages
 * do not describe the activation): g = h Phi(h) with Phi(h) = erfc(-h / sqrt 2) / 2;
 * dh = dg * (Phi(h) + h phi(h)), phi the N(0,1) density.  n elements, contiguous; results are
 * within one bf16 step of the exact values rounded to bf16. */
nvfp4_status nvfp4_gelu_fwd(const void* h, void* g, int64_t n, nvfp4_stream_t stream);
nvfp4_status nvfp4_gelu_bwd(const void* h, const void* dg, void* dh, int64_t n,
                            nvfp4_stream_t stream);

/* The GeLU kernels with the amax of their bf16 output fused in: out[rows][cols] (contiguous) as
 * above, and in ws (reset first) the plain amax and the amax after the 16-point RHT (rht_seed)
 * along rows of out, as nvfp4_amax would compute them from out.  Set the consuming linear
 * context's amax_ready (same ws, same rht_seed) to skip that layer's amax pass.  Shape rules:
 * rows % 16 == 0, cols % 16 == 0. */
nvfp4_status nvfp4_gelu_fwd_amax(const void* h, void* g, int64_t rows, int64_t cols, uint64_t rht_seed,
                                 void* ws, nvfp4_stream_t stream);
nvfp4_status nvfp4_gelu_bwd_amax(const void* h, const void* dg, void* dh, int64_t rows, int64_t cols,
                                 uint64_t rht_seed, void* ws, nvfp4_stream_t stream);

/*
 * nvfp4_quantize without a workspace argument.  The pages have no counterpart: this exists for
 * callers that cannot allocate device memory themselves (a host whose own allocator owns all
 * device memory, or a plugin interface without an allocation hook) and so cannot pass `ws`.
 * Arguments, shape rules and results are those of nvfp4_quantize; the call allocates nothing.
 * Its 256-byte scratch is a fixed device array inside the library, held by every GPU that
 * loads the library until the process exits; a call whose scratch would not fit returns
 * NVFP4_ERR_LIMIT.  The first call on a device looks up the array's device address (do it
 * before any stream capture); that address does not survive cudaDeviceReset of the device.
 * All calls share the array, so calls that overlap on the GPU race; serialise them.
 * Device-side conditions (non-finite input, a wait that ran out of its budget) are kept in the
 * array until nvfp4_poll_noalloc reports them; the output of a flagged call is undefined.
 */
nvfp4_status nvfp4_quantize_noalloc(const void* x, int64_t rows, int64_t cols, int64_t ldx, int along,
                                    nvfp4_round mode, nvfp4_block block, int rht, uint64_t rht_seed,
                                    uint64_t sr_seed, uint32_t stream_id, nvfp4_tensor* out,
                                    nvfp4_stream_t stream);

/* nvfp4_poll for nvfp4_quantize_noalloc (no counterpart in the pages either): synchronize
 * `stream`, then report and clear the flags that the workspace-free calls on the current
 * device left in the library's array, with the precedence of nvfp4_poll.  Allocates nothing. */
nvfp4_status nvfp4_poll_noalloc(nvfp4_stream_t stream);

/*
 * MXFP4, the format the pages compare NVFP4 against (gist.science 2.A: blocks of 32 elements with
 * a power-of-two UE8M0 scale and no tensor scale; 4 "Ergebnisse": MXFP4 needs about 36 % more
 * training tokens to match NVFP4).  One form per call (nvfp4_mx_quantize) or both forms from one
 * read (nvfp4_mx_quantize_dual), a single pass (no tensor amax):
 *   scale code of a block = floor(log2 amax_b) - 2 + 127 clamped to [0, 254] (0 for an all-zero
 *   block), i.e. 2^E with E the block's exponent less that of E2M1's largest value (6 = 1.5 * 2^2);
 *   element u = v * 2^-E, encoded to E2M1 as in nvfp4_quantize (RNE, or SR with the same Philox
 *   fields indexed by the element's position in the form).
 * Layout: codes [rows][k/2] as for NVFP4; scales in 128x4 tiles of 512 bytes, entry (r, kb =
 * k_index/32) at ((r/128)*ceil(k/128) + kb/4)*512 + (r%32)*16 + ((r/32)%4)*4 + kb%4 (zero padding),
 * the layout the tcgen05 kind::mxf4 MMA reads.
 * Shape rules: k % 32 == 0 (k = cols for along = 0, rows for along = 1); along = 1 needs
 * rows % 32 == 0; cols % 16 == 0.  Non-finite inputs are out of contract (not flagged).  ws
 * receives the timeout flag of the tile copies.
 */
typedef struct {
    uint8_t* codes;
    uint8_t* scales;
    int64_t rows;
    int64_t k;
} nvfp4_mx_tensor;

size_t nvfp4_mx_scales_bytes(int64_t rows, int64_t k); /* ceil(rows/128)*128 * ceil(k/128)*4 */
nvfp4_status nvfp4_mx_quantize(const void* x, int64_t rows, int64_t cols, int64_t ldx, int along,
                               nvfp4_round mode, uint64_t sr_seed, uint32_t stream_id,
                               nvfp4_mx_tensor* out, void* ws, nvfp4_stream_t stream);
/* Both MXFP4 forms of x from one read: out_row (along = 0, SR stream stream_row) and out_col
 * (along = 1, SR stream stream_col), each equal to the form nvfp4_mx_quantize gives with the same
 * arguments.  rows % 32 == 0 and cols % 32 == 0; the buffers are the caller's, filled on `stream`;
 * out_row->rows/k and out_col->rows/k are set. */
nvfp4_status nvfp4_mx_quantize_dual(const void* x, int64_t rows, int64_t cols, int64_t ldx, nvfp4_round mode,
                                    uint64_t sr_seed, uint32_t stream_row, uint32_t stream_col,
                                    nvfp4_mx_tensor* out_row, nvfp4_mx_tensor* out_col, void* ws,
                                    nvfp4_stream_t stream);
/* D[M][N] = sum_k A[m][k] * B[n][k] over MXFP4 forms with the same k, by the tcgen05
 * kind::mxf4 block-scaled MMA; fp32 accumulation, bf16 or fp32 output.  Shape rules and kernel
 * choice as nvfp4_gemm (K % 32 == 0). */
nvfp4_status nvfp4_mx_gemm(const nvfp4_mx_tensor* a, const nvfp4_mx_tensor* b, void* d, int64_t ldd,
                           nvfp4_dtype out_dtype, void* ws, nvfp4_stream_t stream);

/*
 * BF16 path for the linear layers the recipe keeps in high precision (gist.science 2.B.1: about
 * 15 % of the linear layers, mostly the last ones, stay in BF16).  The GEMM is the same SM-pair
 * tcgen05 kernel as nvfp4_gemm with kind::f16 MMAs (bf16 operands, fp32 accumulation in TMEM).
 *
 * nvfp4_bf16_gemm: D[M][N] = A[M][K] . B[N][K]^T, A and B bf16 row-major (K-major) with leading
 * dimensions lda, ldb (elements); bf16 or fp32 output.  Shape rules: M, N >= 1; K >= 8, K % 8 == 0;
 * lda >= K, ldb >= K, both % 8 == 0; ldd >= N, ldd * sizeof(out) % 16 == 0.  ws: timeout flag.
 */
nvfp4_status nvfp4_bf16_gemm(const void* a, int64_t lda, const void* b, int64_t ldb, int64_t M, int64_t N,
                             int64_t K, void* d, int64_t ldd, nvfp4_dtype out_dtype, void* ws,
                             nvfp4_stream_t stream);
/* xt[c][r] = x[r][c] for bf16 x[rows][ldx] into xt[cols][ldxt]; rows % 8 == 0, cols % 8 == 0,
 * ldx and ldxt multiples of 8 (elements). */
nvfp4_status nvfp4_bf16_transpose(const void* x, int64_t rows, int64_t cols, int64_t ldx, void* xt,
                                  int64_t ldxt, nvfp4_stream_t stream);
/* The BF16 linear layer y = x w^T (x [T][d], w [n][d], dy [T][n], all bf16 contiguous):
 *   fwd: y [T][n] (bf16) = x . w^T;
 *   bwd: dx [T][d] (bf16) = dy . w and dw [n][d] (fp32) = dy^T . x, through the K-major
 *        transposes w^T, dy^T and x^T written into `scratch` (caller-owned,
 *        nvfp4_linear_bf16_scratch_bytes(T, d, n) bytes, 16-byte aligned).  dx or dw may be NULL.
 * Shape rules: T, d, n positive multiples of 8. */
size_t nvfp4_linear_bf16_scratch_bytes(int64_t T, int64_t d, int64_t n);
nvfp4_status nvfp4_linear_bf16_fwd(const void* x, const void* w, void* y, int64_t T, int64_t d, int64_t n,
                                   void* ws, nvfp4_stream_t stream);
nvfp4_status nvfp4_linear_bf16_bwd(const void* x, const void* w, const void* dy, void* dx, float* dw,
                                   int64_t T, int64_t d, int64_t n, void* scratch, void* ws,
                                   nvfp4_stream_t stream);

/* Synchronize `stream`, then report (and clear) the device flags of `ws`: NVFP4_ERR_TIMEOUT
 * takes precedence over NVFP4_ERR_NONFINITE; NVFP4_OK when neither is set. */
nvfp4_status nvfp4_poll(void* ws, nvfp4_stream_t stream);

/* Device-side wait budget of the GEMM's mbarrier spins, in nanoseconds (default 2e9).
 * Process-wide; 0 restores the default. */
void nvfp4_set_wait_budget_ns(uint64_t ns);

const char* nvfp4_status_string(nvfp4_status s);
int nvfp4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H */
