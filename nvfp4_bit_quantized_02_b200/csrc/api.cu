// api.cu -- the C ABI of libnvfp4 (declared in include/nvfp4.h): argument validation and
// kernel launches.  No allocation, no host synchronisation (except nvfp4_poll), no printing.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>

#include "nvfp4.h"
#include "nvfp4_device.cuh"
#include "nvfp4_internal.h"

using namespace nvfp4;

namespace {

std::atomic<uint64_t> g_budget_ns{2000000000ull};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// sm_100 check, cached per device
nvfp4_status check_device() {
    static std::atomic<int> cached[64];  // 0 unknown, 1 ok, 2 unsupported (any thread may fill it)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (dev < 0 || dev >= 64) return NVFP4_ERR_UNSUPPORTED;
    int c = cached[dev].load(std::memory_order_relaxed);
    if (c == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        c = (major == 10 && minor == 0) ? 1 : 2;
        cached[dev].store(c, std::memory_order_relaxed);
    }
    return c == 1 ? NVFP4_OK : NVFP4_ERR_UNSUPPORTED;
}

nvfp4_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return NVFP4_OK;
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
}

int64_t nkt_of(int64_t k) { return ((k >> 4) + 3) >> 2; }

bool has_scale_padding(int64_t rows, int64_t k) { return (rows & 127) != 0 || ((k >> 4) & 3) != 0; }

nvfp4_status check_form_buffers(const nvfp4_tensor* t, bool need_tiles) {
    if (!t || !t->codes || !t->scales || !t->tensor_scale) return NVFP4_ERR_NULL;
    if (need_tiles && !t->tile_scales) return NVFP4_ERR_NULL;
    if (!aligned16(t->codes) || !aligned16(t->scales)) return NVFP4_ERR_ALIGN;
    return NVFP4_OK;
}

nvfp4_status check_input(const void* x, int64_t rows, int64_t cols, int64_t ld) {
    if (rows < 0 || cols < 0) return NVFP4_ERR_SHAPE;
    if (cols % 16 != 0) return NVFP4_ERR_SHAPE;
    if (ld < cols) return NVFP4_ERR_SHAPE;
    if (rows > 0 && cols > 0) {
        if (!x) return NVFP4_ERR_NULL;
        if (!aligned16(x) || (ld % 8) != 0) return NVFP4_ERR_ALIGN;
    }
    return NVFP4_OK;
}

__global__ void set_f32_kernel(float* p, float v) { *p = v; }

Workspace* ws_of(void* ws) { return reinterpret_cast<Workspace*>(ws); }

cudaError_t reset_amax(void* ws, cudaStream_t s) {
    return cudaMemsetAsync(reinterpret_cast<uint8_t*>(ws) + offsetof(Workspace, amax_a), 0, 2 * sizeof(uint32_t), s);
}

}  // namespace

namespace nvfp4 {

uint32_t rht_signs_host(uint64_t seed) {
    uint32_t c0 = 0, c1 = 0, c2 = NVFP4_STREAM_RHT, c3 = 0;
    uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
    for (int round = 0; round < 10; ++round) {
        const uint64_t p0 = (uint64_t)0xD2511F53u * c0, p1 = (uint64_t)0xCD9E8D57u * c2;
        const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0, n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
        c1 = (uint32_t)p1;
        c3 = (uint32_t)p0;
        c0 = n0;
        c2 = n2;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return c0 & 0xFFFFu;
}

}  // namespace nvfp4

extern "C" {

size_t nvfp4_codes_bytes(int64_t rows, int64_t k) { return (rows > 0 && k > 0) ? (size_t)(rows * (k / 2)) : 0; }

size_t nvfp4_scales_bytes(int64_t rows, int64_t k) {
    if (rows <= 0 || k <= 0) return 0;
    return (size_t)(((rows + 127) / 128) * 128 * nkt_of(k) * 4);
}

size_t nvfp4_tile_scales_bytes(int64_t rows, int64_t k) {
    return (rows > 0 && k > 0) ? (size_t)((rows / 16) * (k / 16)) : 0;
}

size_t nvfp4_workspace_bytes(void) { return sizeof(Workspace); }

nvfp4_status nvfp4_workspace_init(void* ws, nvfp4_stream_t stream) {
    if (!ws) return NVFP4_ERR_WORKSPACE;
    if (nvfp4_status st = check_device()) return st;
    return from_cuda(cudaMemsetAsync(ws, 0, sizeof(Workspace), stream));
}

nvfp4_status nvfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ldx, int along, nvfp4_round mode,
                            nvfp4_block block, int rht, uint64_t rht_seed, uint64_t sr_seed, uint32_t stream_id,
                            nvfp4_tensor* out, void* ws, nvfp4_stream_t stream) {
    if (nvfp4_status st = check_input(x, rows, cols, ldx)) return st;
    if (along != 0 && along != 1) return NVFP4_ERR_ARG;
    if (mode != NVFP4_RNE && mode != NVFP4_SR) return NVFP4_ERR_ARG;
    if (block != NVFP4_BLOCK_1x16 && block != NVFP4_BLOCK_16x16) return NVFP4_ERR_ARG;
    if (rht && (block == NVFP4_BLOCK_16x16 || along == 0)) return NVFP4_ERR_ARG;  // RHT: wgrad (along=1) forms only
    const bool b16 = block == NVFP4_BLOCK_16x16;
    if (nvfp4_status st = check_form_buffers(out, b16)) return st;
    if (!ws) return NVFP4_ERR_WORKSPACE;
    if ((along == 1 || b16) && (rows % 16) != 0) return NVFP4_ERR_SHAPE;
    if (nvfp4_status st = check_device()) return st;
    const int64_t R = along ? cols : rows, K = along ? rows : cols;
    out->rows = R;
    out->k = K;
    out->block = block;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (R == 0 || K == 0) {
        set_f32_kernel<<<1, 1, 0, s>>>(out->tensor_scale, 1.0f);
        return from_cuda(cudaGetLastError());
    }
    Workspace* w = ws_of(ws);
    if (cudaError_t e = reset_amax(ws, s)) return from_cuda(e);
    if (has_scale_padding(R, K))
        if (cudaError_t e = cudaMemsetAsync(out->scales, 0, nvfp4_scales_bytes(R, K), s)) return from_cuda(e);
    const uint32_t signs = rht ? rht_signs_host(rht_seed) : 0u;
    const uint16_t* xb = reinterpret_cast<const uint16_t*>(x);
    cudaError_t e = (along == 1 && rht) ? launch_amax_rht(xb, rows, cols, ldx, signs, &w->amax_a, &w->amax_b, &w->flags, s)
                                        : launch_amax_plain(xb, rows, cols, ldx, &w->amax_a, &w->flags, s);
    if (e != cudaSuccess) return from_cuda(e);
    QuantParams p;
    std::memset(&p, 0, sizeof(p));
    p.x = xb;
    p.rows = rows;
    p.cols = cols;
    p.ld = ldx;
    p.block16 = b16 ? 1 : 0;
    p.signs = signs;
    p.sr_seed = sr_seed;
    p.flags = &w->flags;
    p.row_offset = 0;
    p.rows_total = rows;
    if (along == 0) {
        p.codes_row = out->codes;
        p.scales_row = out->scales;
        p.tiles_row = b16 ? out->tile_scales : nullptr;
        p.st_row = out->tensor_scale;
        p.amax_row = &w->amax_a;
        p.nkt_row = nkt_of(K);
        p.sr_row = mode == NVFP4_SR;
        p.stream_row = stream_id;
    } else {
        p.codes_col = out->codes;
        p.scales_col = out->scales;
        p.tiles_col = b16 ? out->tile_scales : nullptr;
        p.st_col = out->tensor_scale;
        p.amax_col = rht ? &w->amax_b : &w->amax_a;
        p.nkt_col = nkt_of(K);
        p.sr_col = mode == NVFP4_SR;
        p.rht_col = rht ? 1 : 0;
        p.stream_col = stream_id;
    }
    return from_cuda(launch_quantize_tiles(p, s));
}

}  // extern "C"

namespace {

// Both forms of x from one read.  run_amax: pass 1 here (the whole tensor); otherwise the amax
// words already in ws are used (a token shard whose amax the caller has reduced across ranks).
// SR fields are indexed in the forms of the rows_total-row tensor of which x is rows
// [row_offset, row_offset + rows).
nvfp4_status quantize_dual_impl(const void* x, int64_t rows, int64_t cols, int64_t ldx, nvfp4_round mode,
                                uint64_t rht_seed, uint64_t sr_seed, uint32_t stream_row, uint32_t stream_col,
                                nvfp4_tensor* out_row, nvfp4_tensor* out_col, void* ws, nvfp4_stream_t stream,
                                int64_t row_offset, int64_t rows_total, bool run_amax) {
    if (nvfp4_status st = check_input(x, rows, cols, ldx)) return st;
    if (mode != NVFP4_RNE && mode != NVFP4_SR) return NVFP4_ERR_ARG;
    if (nvfp4_status st = check_form_buffers(out_row, false)) return st;
    if (nvfp4_status st = check_form_buffers(out_col, false)) return st;
    if (!ws) return NVFP4_ERR_WORKSPACE;
    if (rows % 16 != 0) return NVFP4_ERR_SHAPE;
    if (row_offset < 0 || row_offset % 16 != 0 || rows_total < row_offset + rows) return NVFP4_ERR_SHAPE;
    if (nvfp4_status st = check_device()) return st;
    out_row->rows = rows;
    out_row->k = cols;
    out_row->block = NVFP4_BLOCK_1x16;
    out_col->rows = cols;
    out_col->k = rows;
    out_col->block = NVFP4_BLOCK_1x16;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (rows == 0 || cols == 0) {
        set_f32_kernel<<<1, 1, 0, s>>>(out_row->tensor_scale, 1.0f);
        set_f32_kernel<<<1, 1, 0, s>>>(out_col->tensor_scale, 1.0f);
        return from_cuda(cudaGetLastError());
    }
    Workspace* w = ws_of(ws);
    if (has_scale_padding(rows, cols))
        if (cudaError_t e = cudaMemsetAsync(out_row->scales, 0, nvfp4_scales_bytes(rows, cols), s)) return from_cuda(e);
    if (has_scale_padding(cols, rows))
        if (cudaError_t e = cudaMemsetAsync(out_col->scales, 0, nvfp4_scales_bytes(cols, rows), s)) return from_cuda(e);
    const uint32_t signs = rht_signs_host(rht_seed);
    const uint16_t* xb = reinterpret_cast<const uint16_t*>(x);
    if (run_amax) {
        if (cudaError_t e = reset_amax(ws, s)) return from_cuda(e);
        if (cudaError_t e = launch_amax_rht(xb, rows, cols, ldx, signs, &w->amax_a, &w->amax_b, &w->flags, s))
            return from_cuda(e);
    }
    QuantParams p;
    std::memset(&p, 0, sizeof(p));
    p.x = xb;
    p.rows = rows;
    p.cols = cols;
    p.ld = ldx;
    p.signs = signs;
    p.sr_seed = sr_seed;
    p.flags = &w->flags;
    p.row_offset = row_offset;
    p.rows_total = rows_total;
    p.codes_row = out_row->codes;
    p.scales_row = out_row->scales;
    p.st_row = out_row->tensor_scale;
    p.amax_row = &w->amax_a;
    p.nkt_row = nkt_of(cols);
    p.sr_row = mode == NVFP4_SR;
    p.stream_row = stream_row;
    p.codes_col = out_col->codes;
    p.scales_col = out_col->scales;
    p.st_col = out_col->tensor_scale;
    p.amax_col = &w->amax_b;
    p.nkt_col = nkt_of(rows);
    p.sr_col = mode == NVFP4_SR;
    p.rht_col = 1;
    p.stream_col = stream_col;
    return from_cuda(launch_quantize_tiles(p, s));
}

}  // namespace

extern "C" {

nvfp4_status nvfp4_quantize_dual(const void* x, int64_t rows, int64_t cols, int64_t ldx, nvfp4_round mode,
                                 uint64_t rht_seed, uint64_t sr_seed, uint32_t stream_row, uint32_t stream_col,
                                 nvfp4_tensor* out_row, nvfp4_tensor* out_col, void* ws, nvfp4_stream_t stream) {
    return quantize_dual_impl(x, rows, cols, ldx, mode, rht_seed, sr_seed, stream_row, stream_col, out_row, out_col, ws,
                              stream, 0, rows, true);
}

nvfp4_status nvfp4_amax(const void* x, int64_t rows, int64_t cols, int64_t ldx, int rht, uint64_t rht_seed, void* ws,
                        nvfp4_stream_t stream) {
    if (nvfp4_status st = check_input(x, rows, cols, ldx)) return st;
    if (!ws) return NVFP4_ERR_WORKSPACE;
    if (rht && rows % 16 != 0) return NVFP4_ERR_SHAPE;
    if (nvfp4_status st = check_device()) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    Workspace* w = ws_of(ws);
    if (cudaError_t e = reset_amax(ws, s)) return from_cuda(e);
    if (rows == 0 || cols == 0) return NVFP4_OK;
    const uint16_t* xb = reinterpret_cast<const uint16_t*>(x);
    return from_cuda(rht ? launch_amax_rht(xb, rows, cols, ldx, rht_signs_host(rht_seed), &w->amax_a, &w->amax_b,
                                           &w->flags, s)
                         : launch_amax_plain(xb, rows, cols, ldx, &w->amax_a, &w->flags, s));
}

size_t nvfp4_workspace_amax_offset(void) { return offsetof(Workspace, amax_a); }

nvfp4_status nvfp4_quantize_dual_shard(const void* x, int64_t rows, int64_t cols, int64_t ldx, int64_t row_offset,
                                       int64_t rows_total, nvfp4_round mode, uint64_t rht_seed, uint64_t sr_seed,
                                       uint32_t stream_row, uint32_t stream_col, nvfp4_tensor* out_row,
                                       nvfp4_tensor* out_col, void* ws, nvfp4_stream_t stream) {
    return quantize_dual_impl(x, rows, cols, ldx, mode, rht_seed, sr_seed, stream_row, stream_col, out_row, out_col, ws,
                              stream, row_offset, rows_total, false);
}

nvfp4_status nvfp4_quantize_weight(const void* wp, int64_t rows, int64_t cols, int64_t ldw, nvfp4_tensor* w_q,
                                   nvfp4_tensor* w_qt, void* ws, nvfp4_stream_t stream) {
    if (nvfp4_status st = check_input(wp, rows, cols, ldw)) return st;
    if (nvfp4_status st = check_form_buffers(w_q, true)) return st;
    if (w_qt)
        if (nvfp4_status st = check_form_buffers(w_qt, false)) return st;
    if (!ws) return NVFP4_ERR_WORKSPACE;
    if (rows % 16 != 0) return NVFP4_ERR_SHAPE;
    if (nvfp4_status st = check_device()) return st;
    w_q->rows = rows;
    w_q->k = cols;
    w_q->block = NVFP4_BLOCK_16x16;
    if (w_qt) {
        w_qt->rows = cols;
        w_qt->k = rows;
        w_qt->block = NVFP4_BLOCK_16x16;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (rows == 0 || cols == 0) {
        set_f32_kernel<<<1, 1, 0, s>>>(w_q->tensor_scale, 1.0f);
        if (w_qt) set_f32_kernel<<<1, 1, 0, s>>>(w_qt->tensor_scale, 1.0f);
        return from_cuda(cudaGetLastError());
    }
    Workspace* w = ws_of(ws);
    if (cudaError_t e = reset_amax(ws, s)) return from_cuda(e);
    if (has_scale_padding(rows, cols))
        if (cudaError_t e = cudaMemsetAsync(w_q->scales, 0, nvfp4_scales_bytes(rows, cols), s)) return from_cuda(e);
    if (w_qt && has_scale_padding(cols, rows))
        if (cudaError_t e = cudaMemsetAsync(w_qt->scales, 0, nvfp4_scales_bytes(cols, rows), s)) return from_cuda(e);
    const uint16_t* xb = reinterpret_cast<const uint16_t*>(wp);
    if (cudaError_t e = launch_amax_plain(xb, rows, cols, ldw, &w->amax_a, &w->flags, s)) return from_cuda(e);
    QuantParams p;
    std::memset(&p, 0, sizeof(p));
    p.x = xb;
    p.rows = rows;
    p.cols = cols;
    p.ld = ldw;
    p.block16 = 1;
    p.flags = &w->flags;
    p.row_offset = 0;
    p.rows_total = rows;
    p.codes_row = w_q->codes;
    p.scales_row = w_q->scales;
    p.tiles_row = w_q->tile_scales;
    p.st_row = w_q->tensor_scale;
    p.amax_row = &w->amax_a;
    p.nkt_row = nkt_of(cols);
    if (w_qt) {
        p.codes_col = w_qt->codes;
        p.scales_col = w_qt->scales;
        p.tiles_col = w_qt->tile_scales;
        p.st_col = w_qt->tensor_scale;
        p.amax_col = &w->amax_a;
        p.nkt_col = nkt_of(rows);
    }
    return from_cuda(launch_quantize_tiles(p, s));
}

nvfp4_status nvfp4_transpose_2d(const nvfp4_tensor* w, nvfp4_tensor* wt, nvfp4_stream_t stream) {
    if (!w || !wt) return NVFP4_ERR_NULL;
    if (nvfp4_status st = check_form_buffers(w, true)) return st;
    if (nvfp4_status st = check_form_buffers(wt, false)) return st;
    if (w->block != NVFP4_BLOCK_16x16) return NVFP4_ERR_ARG;
    const int64_t R = w->rows, K = w->k;
    if (R < 0 || K < 0 || R % 16 || K % 16) return NVFP4_ERR_SHAPE;
    if (nvfp4_status st = check_device()) return st;
    wt->rows = K;
    wt->k = R;
    wt->block = NVFP4_BLOCK_16x16;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (R == 0 || K == 0) {
        set_f32_kernel<<<1, 1, 0, s>>>(wt->tensor_scale, 1.0f);
        return from_cuda(cudaGetLastError());
    }
    if (has_scale_padding(K, R))
        if (cudaError_t e = cudaMemsetAsync(wt->scales, 0, nvfp4_scales_bytes(K, R), s)) return from_cuda(e);
    return from_cuda(launch_transpose_2d(w->codes, w->tile_scales, R, K, wt->codes, wt->scales, wt->tile_scales,
                                         w->tensor_scale, wt->tensor_scale, s));
}

nvfp4_status nvfp4_gemm(const nvfp4_tensor* a, const nvfp4_tensor* b, void* d, int64_t ldd, nvfp4_dtype out_dtype,
                        void* ws, nvfp4_stream_t stream) {
    if (!a || !b || !d) return NVFP4_ERR_NULL;
    if (nvfp4_status st = check_form_buffers(a, false)) return st;
    if (nvfp4_status st = check_form_buffers(b, false)) return st;
    if (!ws) return NVFP4_ERR_WORKSPACE;
    if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_FP32) return NVFP4_ERR_ARG;
    const int64_t M = a->rows, N = b->rows, K = a->k;
    if (b->k != K) return NVFP4_ERR_ARG;
    if (M < 1 || N < 1 || K < 32 || K % 32 != 0) return NVFP4_ERR_SHAPE;
    if (M > (int64_t)1 << 30 || N > (int64_t)1 << 30 || K > (int64_t)1 << 30) return NVFP4_ERR_LIMIT;
    const int64_t esz = out_dtype == NVFP4_OUT_FP32 ? 4 : 2;
    if (ldd < N) return NVFP4_ERR_SHAPE;
    if (!aligned16(d) || (ldd * esz) % 16 != 0) return NVFP4_ERR_ALIGN;
    if (nvfp4_status st = check_device()) return st;
    return from_cuda(launch_gemm_nvf4(a->codes, a->scales, a->tensor_scale, M, b->codes, b->scales, b->tensor_scale, N, K,
                                      d, ldd, out_dtype == NVFP4_OUT_FP32, &ws_of(ws)->flags, g_budget_ns.load(),
                                      reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_gemm_reduce_scatter(const nvfp4_tensor* a, const nvfp4_tensor* b, float* const* shards,
                                       int n_owners, int64_t owner_rows, int64_t ldd, void* ws,
                                       nvfp4_stream_t stream) {
    if (!a || !b || !shards) return NVFP4_ERR_NULL;
    if (nvfp4_status st = check_form_buffers(a, false)) return st;
    if (nvfp4_status st = check_form_buffers(b, false)) return st;
    if (!ws) return NVFP4_ERR_WORKSPACE;
    const int64_t M = a->rows, N = b->rows, K = a->k;
    if (b->k != K) return NVFP4_ERR_ARG;
    if (M < 1 || N < 1 || K < 32 || K % 32 != 0) return NVFP4_ERR_SHAPE;
    if (M > (int64_t)1 << 30 || N > (int64_t)1 << 30 || K > (int64_t)1 << 30) return NVFP4_ERR_LIMIT;
    if (n_owners < 1 || n_owners > 8 || owner_rows < 32 || owner_rows % 32 != 0) return NVFP4_ERR_SHAPE;
    if ((M + owner_rows - 1) / owner_rows != n_owners) return NVFP4_ERR_SHAPE;
    if (ldd < N) return NVFP4_ERR_SHAPE;
    if ((ldd * 4) % 16 != 0) return NVFP4_ERR_ALIGN;
    for (int o = 0; o < n_owners; ++o) {
        if (!shards[o]) return NVFP4_ERR_NULL;
        if (!aligned16(shards[o])) return NVFP4_ERR_ALIGN;
    }
    if (nvfp4_status st = check_device()) return st;
    return from_cuda(launch_gemm_nvf4_reduce_scatter(a->codes, a->scales, a->tensor_scale, M, b->codes, b->scales,
                                                     b->tensor_scale, N, K, shards, n_owners, owner_rows, ldd,
                                                     &ws_of(ws)->flags, g_budget_ns.load(),
                                                     reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_gemm_amax(const nvfp4_tensor* a, const nvfp4_tensor* b, void* d, int64_t ldd, uint64_t rht_seed,
                             void* amax_ws, void* ws, nvfp4_stream_t stream) {
    if (!a || !b || !d) return NVFP4_ERR_NULL;
    if (nvfp4_status st = check_form_buffers(a, false)) return st;
    if (nvfp4_status st = check_form_buffers(b, false)) return st;
    if (!ws || !amax_ws) return NVFP4_ERR_WORKSPACE;
    const int64_t M = a->rows, N = b->rows, K = a->k;
    if (b->k != K) return NVFP4_ERR_ARG;
    if (M < 16 || M % 16 != 0 || N < 1 || K < 32 || K % 32 != 0) return NVFP4_ERR_SHAPE;
    if (M > (int64_t)1 << 30 || N > (int64_t)1 << 30 || K > (int64_t)1 << 30) return NVFP4_ERR_LIMIT;
    if (ldd < N) return NVFP4_ERR_SHAPE;
    if (!aligned16(d) || (ldd * 2) % 16 != 0) return NVFP4_ERR_ALIGN;
    if (nvfp4_status st = check_device()) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaError_t e = reset_amax(amax_ws, s)) return from_cuda(e);
    return from_cuda(launch_gemm_nvf4_amax(a->codes, a->scales, a->tensor_scale, M, b->codes, b->scales, b->tensor_scale, N,
                                           K, d, ldd, &ws_of(amax_ws)->amax_a, rht_signs_host(rht_seed),
                                           &ws_of(ws)->flags, g_budget_ns.load(), s));
}

static nvfp4_status check_ctx(const nvfp4_linear_ctx* c) {
    if (!c) return NVFP4_ERR_NULL;
    if (c->T <= 0 || c->d <= 0 || c->n <= 0) return NVFP4_ERR_SHAPE;
    if (c->T % 64 || c->d % 64 || c->n % 64) return NVFP4_ERR_SHAPE;
    if (!c->ws) return NVFP4_ERR_WORKSPACE;
    return NVFP4_OK;
}

nvfp4_status nvfp4_linear_fwd(const void* x, const void* w, void* y, nvfp4_linear_ctx* ctx, nvfp4_stream_t stream) {
    if (nvfp4_status st = check_ctx(ctx)) return st;
    if (!x || !y || (!w && !ctx->w_cached)) return NVFP4_ERR_NULL;
    // X first: with amax_ready its amax words are in ws, which the weight's quantize overwrites
    const bool ready = ctx->amax_ready != 0;
    ctx->amax_ready = 0;
    nvfp4_status st = quantize_dual_impl(x, ctx->T, ctx->d, ctx->d, NVFP4_RNE, ctx->rht_seed, 0, 0, 0, &ctx->xq,
                                         &ctx->xq_rht, ctx->ws, stream, 0, ctx->T, !ready);
    if (st) return st;
    if (!ctx->w_cached) {
        st = nvfp4_quantize_weight(w, ctx->n, ctx->d, ctx->d, &ctx->wq, &ctx->wqt, ctx->ws, stream);
        if (st) return st;
    }
    if (ctx->y_amax_ws)
        return nvfp4_gemm_amax(&ctx->xq, &ctx->wq, y, ctx->n, ctx->y_rht_seed, ctx->y_amax_ws, ctx->ws, stream);
    return nvfp4_gemm(&ctx->xq, &ctx->wq, y, ctx->n, NVFP4_OUT_BF16, ctx->ws, stream);
}

nvfp4_status nvfp4_linear_bwd(const void* dy, uint64_t sr_seed, void* dx, float* dw, nvfp4_linear_ctx* ctx,
                              nvfp4_stream_t stream) {
    if (nvfp4_status st = check_ctx(ctx)) return st;
    if (!dy) return NVFP4_ERR_NULL;
    const bool ready = ctx->amax_ready != 0;
    ctx->amax_ready = 0;
    nvfp4_status st = quantize_dual_impl(dy, ctx->T, ctx->n, ctx->n, NVFP4_SR, ctx->rht_seed, sr_seed, NVFP4_STREAM_DGRAD,
                                         NVFP4_STREAM_WGRAD, &ctx->dyq, &ctx->dyq_rht, ctx->ws, stream, 0, ctx->T, !ready);
    if (st) return st;
    if (dx) {
        st = ctx->dx_amax_ws ? nvfp4_gemm_amax(&ctx->dyq, &ctx->wqt, dx, ctx->d, ctx->dx_rht_seed, ctx->dx_amax_ws,
                                               ctx->ws, stream)
                             : nvfp4_gemm(&ctx->dyq, &ctx->wqt, dx, ctx->d, NVFP4_OUT_BF16, ctx->ws, stream);
        if (st) return st;
    }
    if (dw) {
        st = nvfp4_gemm(&ctx->dyq_rht, &ctx->xq_rht, dw, ctx->d, NVFP4_OUT_FP32, ctx->ws, stream);
        if (st) return st;
    }
    return NVFP4_OK;
}

nvfp4_status nvfp4_gelu_fwd(const void* h, void* g, int64_t n, nvfp4_stream_t stream) {
    if (n < 0) return NVFP4_ERR_SHAPE;
    if (n == 0) return NVFP4_OK;
    if (!h || !g) return NVFP4_ERR_NULL;
    if (!aligned16(h) || !aligned16(g)) return NVFP4_ERR_ALIGN;
    if (nvfp4_status st = check_device()) return st;
    return from_cuda(launch_gelu_fwd(reinterpret_cast<const uint16_t*>(h), reinterpret_cast<uint16_t*>(g), n,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_gelu_bwd(const void* h, const void* dg, void* dh, int64_t n, nvfp4_stream_t stream) {
    if (n < 0) return NVFP4_ERR_SHAPE;
    if (n == 0) return NVFP4_OK;
    if (!h || !dg || !dh) return NVFP4_ERR_NULL;
    if (!aligned16(h) || !aligned16(dg) || !aligned16(dh)) return NVFP4_ERR_ALIGN;
    if (nvfp4_status st = check_device()) return st;
    return from_cuda(launch_gelu_bwd(reinterpret_cast<const uint16_t*>(h), reinterpret_cast<const uint16_t*>(dg),
                                     reinterpret_cast<uint16_t*>(dh), n, reinterpret_cast<cudaStream_t>(stream)));
}

static nvfp4_status gelu_amax(bool bwd, const void* h, const void* dg, void* out, int64_t rows, int64_t cols,
                              uint64_t rht_seed, void* ws, nvfp4_stream_t stream) {
    if (rows < 0 || cols < 0 || rows % 16 != 0 || cols % 16 != 0) return NVFP4_ERR_SHAPE;
    if (!ws) return NVFP4_ERR_WORKSPACE;
    if (rows > 0 && cols > 0) {
        if (!h || !out || (bwd && !dg)) return NVFP4_ERR_NULL;
        if (!aligned16(h) || !aligned16(out) || (bwd && !aligned16(dg))) return NVFP4_ERR_ALIGN;
    }
    if (nvfp4_status st = check_device()) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaError_t e = reset_amax(ws, s)) return from_cuda(e);
    Workspace* w = ws_of(ws);
    return from_cuda(launch_gelu_amax(bwd, reinterpret_cast<const uint16_t*>(h), reinterpret_cast<const uint16_t*>(dg),
                                      reinterpret_cast<uint16_t*>(out), rows, cols, rht_signs_host(rht_seed), &w->amax_a,
                                      &w->amax_b, &w->flags, s));
}

nvfp4_status nvfp4_gelu_fwd_amax(const void* h, void* g, int64_t rows, int64_t cols, uint64_t rht_seed, void* ws,
                                 nvfp4_stream_t stream) {
    return gelu_amax(false, h, nullptr, g, rows, cols, rht_seed, ws, stream);
}

nvfp4_status nvfp4_gelu_bwd_amax(const void* h, const void* dg, void* dh, int64_t rows, int64_t cols, uint64_t rht_seed,
                                 void* ws, nvfp4_stream_t stream) {
    return gelu_amax(true, h, dg, dh, rows, cols, rht_seed, ws, stream);
}

size_t nvfp4_mx_scales_bytes(int64_t rows, int64_t k) {
    if (rows <= 0 || k <= 0) return 0;
    return (size_t)(((rows + 127) / 128) * 128 * ((k + 127) / 128) * 4);
}

static nvfp4_status check_mx_out(const nvfp4_mx_tensor* out) {
    if (!out || !out->codes || !out->scales) return NVFP4_ERR_NULL;
    if (!aligned16(out->codes) || !aligned16(out->scales)) return NVFP4_ERR_ALIGN;
    return NVFP4_OK;
}

// zero a form's scale tiles where the kernel leaves padding unwritten (R or K/32 ragged)
static cudaError_t clear_mx_padding(const nvfp4_mx_tensor* out, int64_t R, int64_t K, cudaStream_t s) {
    if ((R & 127) != 0 || ((K >> 5) & 3) != 0) return cudaMemsetAsync(out->scales, 0, nvfp4_mx_scales_bytes(R, K), s);
    return cudaSuccess;
}

nvfp4_status nvfp4_mx_quantize(const void* x, int64_t rows, int64_t cols, int64_t ldx, int along, nvfp4_round mode,
                               uint64_t sr_seed, uint32_t stream_id, nvfp4_mx_tensor* out, void* ws,
                               nvfp4_stream_t stream) {
    if (nvfp4_status st = check_input(x, rows, cols, ldx)) return st;
    if (along != 0 && along != 1) return NVFP4_ERR_ARG;
    if (mode != NVFP4_RNE && mode != NVFP4_SR) return NVFP4_ERR_ARG;
    if (nvfp4_status st = check_mx_out(out)) return st;
    if (!ws) return NVFP4_ERR_WORKSPACE;
    const int64_t R = along ? cols : rows, K = along ? rows : cols;
    if (K % 32 != 0) return NVFP4_ERR_SHAPE;
    if (nvfp4_status st = check_device()) return st;
    out->rows = R;
    out->k = K;
    if (R == 0 || K == 0) return NVFP4_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaError_t e = clear_mx_padding(out, R, K, s)) return from_cuda(e);
    MxParams p;
    std::memset(&p, 0, sizeof(p));
    p.x = reinterpret_cast<const uint16_t*>(x);
    p.rows = rows;
    p.cols = cols;
    p.ld = ldx;
    if (along == 0) {
        p.codes = out->codes;
        p.scales = out->scales;
        p.nkt = (K + 127) / 128;
        p.stream_id = stream_id;
    } else {
        p.codes_col = out->codes;
        p.scales_col = out->scales;
        p.nkt_col = (K + 127) / 128;
        p.stream_col = stream_id;
    }
    p.sr = mode == NVFP4_SR;
    p.flags = &ws_of(ws)->flags;
    return from_cuda(launch_quantize_mx(p, along == 0, along == 1, sr_seed, s));
}

nvfp4_status nvfp4_mx_quantize_dual(const void* x, int64_t rows, int64_t cols, int64_t ldx, nvfp4_round mode,
                                    uint64_t sr_seed, uint32_t stream_row, uint32_t stream_col,
                                    nvfp4_mx_tensor* out_row, nvfp4_mx_tensor* out_col, void* ws,
                                    nvfp4_stream_t stream) {
    if (nvfp4_status st = check_input(x, rows, cols, ldx)) return st;
    if (mode != NVFP4_RNE && mode != NVFP4_SR) return NVFP4_ERR_ARG;
    if (nvfp4_status st = check_mx_out(out_row)) return st;
    if (nvfp4_status st = check_mx_out(out_col)) return st;
    if (!ws) return NVFP4_ERR_WORKSPACE;
    if (rows % 32 != 0 || cols % 32 != 0) return NVFP4_ERR_SHAPE;
    if (nvfp4_status st = check_device()) return st;
    out_row->rows = rows;
    out_row->k = cols;
    out_col->rows = cols;
    out_col->k = rows;
    if (rows == 0 || cols == 0) return NVFP4_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaError_t e = clear_mx_padding(out_row, rows, cols, s)) return from_cuda(e);
    if (cudaError_t e = clear_mx_padding(out_col, cols, rows, s)) return from_cuda(e);
    MxParams p;
    std::memset(&p, 0, sizeof(p));
    p.x = reinterpret_cast<const uint16_t*>(x);
    p.rows = rows;
    p.cols = cols;
    p.ld = ldx;
    p.codes = out_row->codes;
    p.scales = out_row->scales;
    p.nkt = (cols + 127) / 128;
    p.stream_id = stream_row;
    p.codes_col = out_col->codes;
    p.scales_col = out_col->scales;
    p.nkt_col = (rows + 127) / 128;
    p.stream_col = stream_col;
    p.sr = mode == NVFP4_SR;
    p.flags = &ws_of(ws)->flags;
    return from_cuda(launch_quantize_mx(p, true, true, sr_seed, s));
}

nvfp4_status nvfp4_mx_gemm(const nvfp4_mx_tensor* a, const nvfp4_mx_tensor* b, void* d, int64_t ldd,
                           nvfp4_dtype out_dtype, void* ws, nvfp4_stream_t stream) {
    if (!a || !b || !d || !a->codes || !a->scales || !b->codes || !b->scales) return NVFP4_ERR_NULL;
    if (!aligned16(a->codes) || !aligned16(a->scales) || !aligned16(b->codes) || !aligned16(b->scales))
        return NVFP4_ERR_ALIGN;
    if (!ws) return NVFP4_ERR_WORKSPACE;
    if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_FP32) return NVFP4_ERR_ARG;
    const int64_t M = a->rows, N = b->rows, K = a->k;
    if (b->k != K) return NVFP4_ERR_ARG;
    if (M < 1 || N < 1 || K < 32 || K % 32 != 0) return NVFP4_ERR_SHAPE;
    if (M > (int64_t)1 << 30 || N > (int64_t)1 << 30 || K > (int64_t)1 << 30) return NVFP4_ERR_LIMIT;
    const int64_t esz = out_dtype == NVFP4_OUT_FP32 ? 4 : 2;
    if (ldd < N) return NVFP4_ERR_SHAPE;
    if (!aligned16(d) || (ldd * esz) % 16 != 0) return NVFP4_ERR_ALIGN;
    if (nvfp4_status st = check_device()) return st;
    return from_cuda(launch_gemm_mxf4(a->codes, a->scales, M, b->codes, b->scales, N, K, d, ldd,
                                      out_dtype == NVFP4_OUT_FP32, &ws_of(ws)->flags, g_budget_ns.load(),
                                      reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_bf16_gemm(const void* a, int64_t lda, const void* b, int64_t ldb, int64_t M, int64_t N, int64_t K,
                             void* d, int64_t ldd, nvfp4_dtype out_dtype, void* ws, nvfp4_stream_t stream) {
    if (!a || !b || !d) return NVFP4_ERR_NULL;
    if (!ws) return NVFP4_ERR_WORKSPACE;
    if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_FP32) return NVFP4_ERR_ARG;
    if (M < 1 || N < 1 || K < 8 || K % 8 != 0 || lda < K || ldb < K) return NVFP4_ERR_SHAPE;
    if (M > (int64_t)1 << 30 || N > (int64_t)1 << 30 || K > (int64_t)1 << 30) return NVFP4_ERR_LIMIT;
    const int64_t esz = out_dtype == NVFP4_OUT_FP32 ? 4 : 2;
    if (ldd < N) return NVFP4_ERR_SHAPE;
    if (!aligned16(a) || !aligned16(b) || !aligned16(d) || lda % 8 || ldb % 8 || (ldd * esz) % 16) return NVFP4_ERR_ALIGN;
    if (nvfp4_status st = check_device()) return st;
    return from_cuda(launch_gemm_bf16(reinterpret_cast<const uint16_t*>(a), lda, reinterpret_cast<const uint16_t*>(b), ldb,
                                      M, N, K, d, ldd, out_dtype == NVFP4_OUT_FP32, &ws_of(ws)->flags, g_budget_ns.load(),
                                      reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_bf16_transpose(const void* x, int64_t rows, int64_t cols, int64_t ldx, void* xt, int64_t ldxt,
                                  nvfp4_stream_t stream) {
    if (rows < 0 || cols < 0 || rows % 8 || cols % 8 || ldx < cols || ldxt < rows) return NVFP4_ERR_SHAPE;
    if (rows == 0 || cols == 0) return NVFP4_OK;
    if (!x || !xt) return NVFP4_ERR_NULL;
    if (!aligned16(x) || !aligned16(xt) || ldx % 8 || ldxt % 8) return NVFP4_ERR_ALIGN;
    if (nvfp4_status st = check_device()) return st;
    return from_cuda(launch_transpose_bf16(reinterpret_cast<const uint16_t*>(x), rows, cols, ldx,
                                           reinterpret_cast<uint16_t*>(xt), ldxt, reinterpret_cast<cudaStream_t>(stream)));
}

size_t nvfp4_linear_bf16_scratch_bytes(int64_t T, int64_t d, int64_t n) {
    if (T <= 0 || d <= 0 || n <= 0) return 0;
    return (size_t)(2 * (d * n + n * T + d * T));
}

nvfp4_status nvfp4_linear_bf16_fwd(const void* x, const void* w, void* y, int64_t T, int64_t d, int64_t n, void* ws,
                                   nvfp4_stream_t stream) {
    if (T <= 0 || d <= 0 || n <= 0 || T % 8 || d % 8 || n % 8) return NVFP4_ERR_SHAPE;
    return nvfp4_bf16_gemm(x, d, w, d, T, n, d, y, n, NVFP4_OUT_BF16, ws, stream);
}

nvfp4_status nvfp4_linear_bf16_bwd(const void* x, const void* w, const void* dy, void* dx, float* dw, int64_t T,
                                   int64_t d, int64_t n, void* scratch, void* ws, nvfp4_stream_t stream) {
    if (T <= 0 || d <= 0 || n <= 0 || T % 8 || d % 8 || n % 8) return NVFP4_ERR_SHAPE;
    if (!x || !w || !dy || !scratch) return NVFP4_ERR_NULL;
    if (!aligned16(scratch)) return NVFP4_ERR_ALIGN;
    uint16_t* wt = reinterpret_cast<uint16_t*>(scratch);   // [d][n]
    uint16_t* dyt = wt + d * n;                             // [n][T]
    uint16_t* xt = dyt + n * T;                             // [d][T]
    if (dx) {
        if (nvfp4_status st = nvfp4_bf16_transpose(w, n, d, d, wt, n, stream)) return st;
        if (nvfp4_status st = nvfp4_bf16_gemm(dy, n, wt, n, T, d, n, dx, d, NVFP4_OUT_BF16, ws, stream)) return st;
    }
    if (dw) {
        if (nvfp4_status st = nvfp4_bf16_transpose(dy, T, n, n, dyt, T, stream)) return st;
        if (nvfp4_status st = nvfp4_bf16_transpose(x, T, d, d, xt, T, stream)) return st;
        if (nvfp4_status st = nvfp4_bf16_gemm(dyt, T, xt, T, n, d, T, dw, d, NVFP4_OUT_FP32, ws, stream)) return st;
    }
    return NVFP4_OK;
}

nvfp4_status nvfp4_poll(void* ws, nvfp4_stream_t stream) {
    if (!ws) return NVFP4_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return from_cuda(cudaErrorUnknown);
    uint32_t flags = 0;
    if (cudaMemcpy(&flags, ws, sizeof(flags), cudaMemcpyDeviceToHost) != cudaSuccess) return from_cuda(cudaErrorUnknown);
    if (flags && cudaMemset(ws, 0, sizeof(uint32_t)) != cudaSuccess) return from_cuda(cudaErrorUnknown);
    if (flags & kFlagTimeout) return NVFP4_ERR_TIMEOUT;
    if (flags & kFlagNonFinite) return NVFP4_ERR_NONFINITE;
    return NVFP4_OK;
}

void nvfp4_set_wait_budget_ns(uint64_t ns) { g_budget_ns.store(ns ? ns : 2000000000ull); }

const char* nvfp4_status_string(nvfp4_status s) {
    switch (s) {
        case NVFP4_OK: return "ok";
        case NVFP4_ERR_NULL: return "a required pointer is NULL";
        case NVFP4_ERR_ALIGN: return "a pointer or leading dimension is not 16-byte aligned";
        case NVFP4_ERR_SHAPE: return "a size violates the call's shape rule";
        case NVFP4_ERR_ARG: return "an argument is out of range or operands are inconsistent";
        case NVFP4_ERR_WORKSPACE: return "workspace missing";
        case NVFP4_ERR_CUDA: return "a CUDA launch or runtime call failed";
        case NVFP4_ERR_NONFINITE: return "NaN or Inf in a quantized input";
        case NVFP4_ERR_TIMEOUT: return "a device-side wait ran out of its time budget";
        case NVFP4_ERR_UNSUPPORTED: return "device is not sm_100 (B200)";
        case NVFP4_ERR_LIMIT: return "a size exceeds a fixed limit of the call";
    }
    return "unknown status";
}

int nvfp4_version(void) { return 1; }

}  // extern "C"
