// nvfp4_internal.h -- declarations shared by the CUDA translation units of libnvfp4.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace nvfp4 {

// workspace layout (256 bytes, caller-owned device memory)
struct Workspace {
    uint32_t flags;       // kFlag* bits, sticky until nvfp4_poll
    uint32_t amax_a;      // fp32 bits: plain amax of the last quantize call
    uint32_t amax_b;      // fp32 bits: amax after the RHT
    uint32_t pad[61];
};
static_assert(sizeof(Workspace) == 256, "workspace is 256 bytes");

constexpr uint32_t kFlagNonFinite = 1u;
constexpr uint32_t kFlagTimeout = 2u;

// the 16 RHT signs as bf16-pair masks (0x80008000 for a -1 sign), a by-value kernel parameter
struct SignMasks {
    uint32_t m[16];
};
inline SignMasks sign_masks(uint32_t signs) {
    SignMasks s;
    for (int j = 0; j < 16; ++j) s.m[j] = ((signs >> j) & 1u) ? 0x80008000u : 0u;
    return s;
}

// parameters of the tile quantizer (one read of x, up to two forms)
struct QuantParams {
    const uint16_t* x;
    int64_t rows, cols, ld;
    int32_t block16;  // 1: 16x16 tiles (both forms share the tile scale)
    // ROW form: K = cols
    uint8_t* codes_row;
    uint8_t* scales_row;
    uint8_t* tiles_row;
    float* st_row;
    const uint32_t* amax_row;
    int64_t nkt_row;
    int32_t sr_row;
    uint32_t stream_row;
    // COL form: K = rows (the transposed operand)
    uint8_t* codes_col;
    uint8_t* scales_col;
    uint8_t* tiles_col;
    float* st_col;
    const uint32_t* amax_col;
    int64_t nkt_col;
    int32_t sr_col;
    int32_t rht_col;
    uint32_t stream_col;
    uint32_t signs;
    uint64_t sr_seed;
    uint32_t* flags;  // workspace flags (timeout of a tile copy)
    // filled by launch_quantize_tiles (constant-bank operands in the kernel):
    uint32_t sign_mask2[16];  // RHT sign j as a bf16-pair mask: 0x80008000 when sign j is -1, else 0
    uint32_t key0[10];        // Philox4x32-10 round keys of sr_seed (Weyl sequence of its two words)
    uint32_t key1[10];
    // SR bit indexing of a token shard: x holds rows [row_offset, row_offset + rows) of a
    // rows_total-row tensor, and SR fields are indexed in the forms of that whole tensor
    int64_t row_offset;
    int64_t rows_total;
};

// parameters of the MXFP4 tile quantizer (one form per call)
struct MxParams {
    const uint16_t* x;
    int64_t rows, cols, ld;    // the bf16 source [rows][ld]
    // the row form (K = cols) and the column form (K = rows); a call fills the forms it launches
    uint8_t* codes;            // row form's codes [rows][cols/2]
    uint8_t* scales;           // its UE8M0 scales in 128x4 tiles
    int64_t nkt;               // ceil(cols / 128): 128x4 scale tiles per 128 form rows
    uint32_t stream_id;        // its SR stream
    uint8_t* codes_col;        // column form's codes [cols][rows/2]
    uint8_t* scales_col;
    int64_t nkt_col;           // ceil(rows / 128)
    uint32_t stream_col;
    int32_t sr;                // 1: stochastic rounding (both forms)
    uint32_t* flags;           // workspace flags (timeout of a tile copy)
    uint32_t key0[10];         // Philox4x32-10 round keys of the SR seed
    uint32_t key1[10];
};

cudaError_t launch_quantize_mx(const MxParams& p, bool row_form, bool column_form, uint64_t sr_seed, cudaStream_t s);

cudaError_t launch_amax_plain(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, uint32_t* amax,
                              uint32_t* flags, cudaStream_t s);
cudaError_t launch_amax_rht(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, uint32_t signs,
                            uint32_t* amax_plain, uint32_t* amax_rht, uint32_t* flags, cudaStream_t s);
cudaError_t launch_quantize_tiles(const QuantParams& p, cudaStream_t s);
cudaError_t launch_transpose_2d(const uint8_t* codes, const uint8_t* tiles, int64_t R, int64_t K, uint8_t* codes_t,
                                uint8_t* scales_t, uint8_t* tiles_t, const float* st_in, float* st_out,
                                cudaStream_t s);
cudaError_t launch_gemm_nvf4(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_st, int64_t M,
                             const uint8_t* b_codes, const uint8_t* b_scales, const float* b_st, int64_t N, int64_t K,
                             void* d, int64_t ldd, bool out_fp32, uint32_t* flags, uint64_t budget_ns,
                             cudaStream_t stream);
cudaError_t launch_gemm_nvf4_reduce_scatter(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_st, int64_t M,
                                            const uint8_t* b_codes, const uint8_t* b_scales, const float* b_st, int64_t N,
                                            int64_t K, float* const* shards, int n_owners, int64_t owner_rows, int64_t ldd,
                                            uint32_t* flags, uint64_t budget_ns, cudaStream_t stream);
cudaError_t launch_gemm_nvf4_amax(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_st, int64_t M,
                                  const uint8_t* b_codes, const uint8_t* b_scales, const float* b_st, int64_t N, int64_t K,
                                  void* d, int64_t ldd, uint32_t* amax_out, uint32_t rht_signs, uint32_t* flags,
                                  uint64_t budget_ns, cudaStream_t stream);
cudaError_t launch_gemm_mxf4(const uint8_t* a_codes, const uint8_t* a_scales, int64_t M, const uint8_t* b_codes,
                             const uint8_t* b_scales, int64_t N, int64_t K, void* d, int64_t ldd, bool out_fp32,
                             uint32_t* flags, uint64_t budget_ns, cudaStream_t stream);
cudaError_t launch_gemm_bf16(const uint16_t* a, int64_t lda, const uint16_t* b, int64_t ldb, int64_t M, int64_t N,
                             int64_t K, void* d, int64_t ldd, bool out_fp32, uint32_t* flags, uint64_t budget_ns,
                             cudaStream_t stream);
cudaError_t launch_transpose_bf16(const uint16_t* x, int64_t rows, int64_t cols, int64_t ldx, uint16_t* xt, int64_t ldt,
                                  cudaStream_t s);
cudaError_t launch_gelu_fwd(const uint16_t* h, uint16_t* g, int64_t n, cudaStream_t s);
cudaError_t launch_gelu_bwd(const uint16_t* h, const uint16_t* dg, uint16_t* dh, int64_t n, cudaStream_t s);
cudaError_t launch_gelu_amax(bool bwd, const uint16_t* h, const uint16_t* dg, uint16_t* out, int64_t rows,
                             int64_t cols, uint32_t signs, uint32_t* amax_plain, uint32_t* amax_rht, uint32_t* flags,
                             cudaStream_t s);

// host-side Philox4x32-10 (same algorithm as the device one) for the RHT sign draw
uint32_t rht_signs_host(uint64_t seed);

}  // namespace nvfp4
