"""Python binding of libnvfp4 (include/nvfp4.h): NVFP4 quantization and block-scaled FP4 GEMMs
for the fprop, dgrad and wgrad GEMMs of a linear layer on a B200 (sm_100a).

Argument marshalling only: every step of the path runs in the CUDA kernels of
``libnvfp4.so``.  PyTorch provides device memory and the current stream.  Importing this
module does not load the library; the first call does, and raises if it is missing -- there is
no CPU fallback.

The functions carry the C names: ``nvfp4_quantize``, ``nvfp4_quantize_dual``,
``nvfp4_quantize_weight``, ``nvfp4_transpose_2d``, ``nvfp4_gemm``, ``nvfp4_linear_fwd``,
``nvfp4_linear_bwd``, ``nvfp4_gelu_fwd``, ``nvfp4_gelu_bwd``, ``nvfp4_poll``, and for data-parallel
token shards ``nvfp4_amax``, ``nvfp4_quantize_dual_shard`` (and ``nvfp4_quantize_dual_dp``, which
all-reduces the amax between them).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4.so")

RNE, SR = 0, 1
BLOCK_1x16, BLOCK_16x16 = 0, 1
OUT_BF16, OUT_FP32 = 0, 1
STREAM_DGRAD, STREAM_WGRAD, STREAM_RHT = 1, 2, 3

STATUS = {0: "OK", 1: "ERR_NULL", 2: "ERR_ALIGN", 3: "ERR_SHAPE", 4: "ERR_ARG", 5: "ERR_WORKSPACE", 6: "ERR_CUDA",
          7: "ERR_NONFINITE", 8: "ERR_TIMEOUT", 9: "ERR_UNSUPPORTED", 10: "ERR_LIMIT"}


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({_lib().nvfp4_status_string(status).decode()})")


class CTensor(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("tile_scales", ctypes.c_void_p),
                ("tensor_scale", ctypes.c_void_p), ("rows", ctypes.c_int64), ("k", ctypes.c_int64),
                ("block", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class CMXTensor(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("rows", ctypes.c_int64), ("k", ctypes.c_int64)]


class CLinearCtx(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int64), ("n", ctypes.c_int64), ("rht_seed", ctypes.c_uint64),
                ("xq", CTensor), ("xq_rht", CTensor), ("wq", CTensor), ("wqt", CTensor), ("dyq", CTensor),
                ("dyq_rht", CTensor), ("ws", ctypes.c_void_p), ("w_cached", ctypes.c_int32),
                ("amax_ready", ctypes.c_int32), ("y_amax_ws", ctypes.c_void_p), ("y_rht_seed", ctypes.c_uint64),
                ("dx_amax_ws", ctypes.c_void_p), ("dx_rht_seed", ctypes.c_uint64)]


_L = None


def _lib():
    global _L
    if _L is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libnvfp4.so is not built ({LIB_PATH}); run __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        c = ctypes
        vp, i64, u64, u32, i32 = c.c_void_p, c.c_int64, c.c_uint64, c.c_uint32, c.c_int
        T = c.POINTER(CTensor)
        sig = {
            "nvfp4_codes_bytes": ([i64, i64], c.c_size_t),
            "nvfp4_scales_bytes": ([i64, i64], c.c_size_t),
            "nvfp4_tile_scales_bytes": ([i64, i64], c.c_size_t),
            "nvfp4_workspace_bytes": ([], c.c_size_t),
            "nvfp4_workspace_init": ([vp, vp], i32),
            "nvfp4_quantize": ([vp, i64, i64, i64, i32, i32, i32, i32, u64, u64, u32, T, vp, vp], i32),
            "nvfp4_quantize_dual": ([vp, i64, i64, i64, i32, u64, u64, u32, u32, T, T, vp, vp], i32),
            "nvfp4_quantize_weight": ([vp, i64, i64, i64, T, T, vp, vp], i32),
            "nvfp4_amax": ([vp, i64, i64, i64, i32, u64, vp, vp], i32),
            "nvfp4_workspace_amax_offset": ([], c.c_size_t),
            "nvfp4_quantize_dual_shard": ([vp, i64, i64, i64, i64, i64, i32, u64, u64, u32, u32, T, T, vp, vp], i32),
            "nvfp4_transpose_2d": ([T, T, vp], i32),
            "nvfp4_gemm": ([T, T, vp, i64, i32, vp, vp], i32),
            "nvfp4_gemm_reduce_scatter": ([T, T, c.POINTER(vp), i32, i64, i64, vp, vp], i32),
            "nvfp4_gemm_amax": ([T, T, vp, i64, u64, vp, vp, vp], i32),
            "nvfp4_linear_fwd": ([vp, vp, vp, c.POINTER(CLinearCtx), vp], i32),
            "nvfp4_linear_bwd": ([vp, u64, vp, vp, c.POINTER(CLinearCtx), vp], i32),
            "nvfp4_gelu_fwd": ([vp, vp, i64, vp], i32),
            "nvfp4_gelu_bwd": ([vp, vp, vp, i64, vp], i32),
            "nvfp4_gelu_fwd_amax": ([vp, vp, i64, i64, u64, vp, vp], i32),
            "nvfp4_gelu_bwd_amax": ([vp, vp, vp, i64, i64, u64, vp, vp], i32),
            "nvfp4_poll": ([vp, vp], i32),
            "nvfp4_mx_scales_bytes": ([i64, i64], c.c_size_t),
            "nvfp4_bf16_gemm": ([vp, i64, vp, i64, i64, i64, i64, vp, i64, i32, vp, vp], i32),
            "nvfp4_bf16_transpose": ([vp, i64, i64, i64, vp, i64, vp], i32),
            "nvfp4_linear_bf16_scratch_bytes": ([i64, i64, i64], c.c_size_t),
            "nvfp4_linear_bf16_fwd": ([vp, vp, vp, i64, i64, i64, vp, vp], i32),
            "nvfp4_linear_bf16_bwd": ([vp, vp, vp, vp, vp, i64, i64, i64, vp, vp, vp], i32),
            "nvfp4_mx_quantize": ([vp, i64, i64, i64, i32, i32, u64, u32, c.POINTER(CMXTensor), vp, vp], i32),
            "nvfp4_mx_quantize_dual": ([vp, i64, i64, i64, i32, u64, u32, u32, c.POINTER(CMXTensor),
                                        c.POINTER(CMXTensor), vp, vp], i32),
            "nvfp4_mx_gemm": ([c.POINTER(CMXTensor), c.POINTER(CMXTensor), vp, i64, i32, vp, vp], i32),
            "nvfp4_quantize_noalloc": ([vp, i64, i64, i64, i32, i32, i32, i32, u64, u64, u32, T, vp], i32),
            "nvfp4_poll_noalloc": ([vp], i32),
            "nvfp4_set_wait_budget_ns": ([u64], None),
            "nvfp4_status_string": ([i32], c.c_char_p),
            "nvfp4_version": ([], i32),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _L = L
    return _L


def lib():
    """The loaded ctypes library (raises ImportError if it is not built)."""
    return _lib()


def _check(status: int, what: str):
    if status != 0:
        raise NVFP4Error(status, what)


# the current stream's raw handle without building a Stream object (a tenth of the cost, which
# matters for small calls); the public route where this torch does not offer it
_RAW_STREAM = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream=None):
    if stream is not None:
        return stream.cuda_stream
    if _RAW_STREAM is not None:
        return _RAW_STREAM(torch.cuda.current_device())
    return torch.cuda.current_stream().cuda_stream


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


# ---------------------------------------------------------------------------------------
# workspace
# ---------------------------------------------------------------------------------------
class Workspace:
    """256 bytes of device memory for amax slots and the sticky device flags."""

    def __init__(self, device=None):
        device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.buf = torch.empty(_lib().nvfp4_workspace_bytes(), dtype=torch.uint8, device=device)
        _check(_lib().nvfp4_workspace_init(_ptr(self.buf), _stream()), "nvfp4_workspace_init")

    @property
    def ptr(self):
        return _ptr(self.buf)

    def amax_words(self) -> torch.Tensor:
        """The two amax words (plain, after the RHT) as an int32 view of the device buffer: fp32
        bit patterns of non-negative values, so an integer MAX reduction is exact."""
        off = _lib().nvfp4_workspace_amax_offset()
        return self.buf[off:off + 8].view(torch.int32)


_DEFAULT_WS = {}


def default_workspace() -> Workspace:
    dev = torch.cuda.current_device()
    if dev not in _DEFAULT_WS:
        _DEFAULT_WS[dev] = Workspace()
    return _DEFAULT_WS[dev]


def nvfp4_poll(ws: Workspace | None = None, stream=None) -> int:
    """Synchronize the stream and return (and clear) the workspace's device status."""
    ws = ws or default_workspace()
    return _lib().nvfp4_poll(ws.ptr, _stream(stream))


def nvfp4_set_wait_budget_ns(ns: int):
    _lib().nvfp4_set_wait_budget_ns(int(ns))


# ---------------------------------------------------------------------------------------
# quantized operand forms
# ---------------------------------------------------------------------------------------
@dataclass
class NVFP4Tensor:
    """One quantized operand form (device buffers owned by torch)."""
    codes: torch.Tensor          # uint8 [rows][k/2]
    scales: torch.Tensor         # uint8, 128x4-tile swizzled E4M3 block scales
    tile_scales: torch.Tensor | None  # uint8 [rows/16][k/16] for 16x16 forms
    tensor_scale: torch.Tensor   # float32 [1]: decode scale s_t
    rows: int
    k: int
    block: int

    @staticmethod
    def empty(rows: int, k: int, block: int = BLOCK_1x16, device=None) -> "NVFP4Tensor":
        L = _lib()
        device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        codes = torch.empty(max(L.nvfp4_codes_bytes(rows, k), 1), dtype=torch.uint8, device=device)
        scales = torch.empty(max(L.nvfp4_scales_bytes(rows, k), 16), dtype=torch.uint8, device=device)
        tiles = None
        if block == BLOCK_16x16:
            tiles = torch.empty(max(L.nvfp4_tile_scales_bytes(rows, k), 1), dtype=torch.uint8, device=device)
        st = torch.empty(1, dtype=torch.float32, device=device)
        return NVFP4Tensor(codes, scales, tiles, st, rows, k, block)

    def c(self) -> CTensor:
        return CTensor(self.codes.data_ptr(), self.scales.data_ptr(),
                       self.tile_scales.data_ptr() if self.tile_scales is not None else None,
                       self.tensor_scale.data_ptr(), self.rows, self.k, self.block, 0)

    def codes_2d(self) -> torch.Tensor:
        return self.codes[: self.rows * (self.k // 2)].view(self.rows, self.k // 2)


def _bf16_2d(x: torch.Tensor):
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise TypeError("expected a 2-D bf16 CUDA tensor")
    if x.stride(1) != 1:
        raise ValueError("inner dimension must be contiguous")
    return x.shape[0], x.shape[1], x.stride(0)


def nvfp4_quantize(x: torch.Tensor, along: int = 0, mode: int = RNE, block: int = BLOCK_1x16, rht: bool = False,
                   rht_seed: int = 0, sr_seed: int = 0, stream_id: int = 0, out: NVFP4Tensor | None = None,
                   ws: Workspace | None = None, stream=None) -> NVFP4Tensor:
    rows, cols, ld = _bf16_2d(x)
    R, K = (cols, rows) if along else (rows, cols)
    out = out or NVFP4Tensor.empty(R, K, block, x.device)
    ws = ws or default_workspace()
    ct = out.c()
    st = _lib().nvfp4_quantize(_ptr(x), rows, cols, ld, along, mode, block, int(rht), rht_seed, sr_seed, stream_id,
                               ctypes.byref(ct), ws.ptr, _stream(stream))
    _check(st, "nvfp4_quantize")
    return out


def nvfp4_quantize_dual(x: torch.Tensor, mode: int = RNE, rht_seed: int = 0, sr_seed: int = 0, stream_row: int = 0,
                        stream_col: int = 0, out_row: NVFP4Tensor | None = None, out_col: NVFP4Tensor | None = None,
                        ws: Workspace | None = None, stream=None):
    rows, cols, ld = _bf16_2d(x)
    out_row = out_row or NVFP4Tensor.empty(rows, cols, BLOCK_1x16, x.device)
    out_col = out_col or NVFP4Tensor.empty(cols, rows, BLOCK_1x16, x.device)
    ws = ws or default_workspace()
    a, b = out_row.c(), out_col.c()
    st = _lib().nvfp4_quantize_dual(_ptr(x), rows, cols, ld, mode, rht_seed, sr_seed, stream_row, stream_col,
                                    ctypes.byref(a), ctypes.byref(b), ws.ptr, _stream(stream))
    _check(st, "nvfp4_quantize_dual")
    return out_row, out_col


def nvfp4_amax(x: torch.Tensor, rht: bool = True, rht_seed: int = 0, ws: Workspace | None = None,
               stream=None) -> Workspace:
    """Pass 1 alone: the amax of x (plain, and after the RHT along rows when rht) into ws."""
    rows, cols, ld = _bf16_2d(x)
    ws = ws or default_workspace()
    _check(_lib().nvfp4_amax(_ptr(x), rows, cols, ld, 1 if rht else 0, rht_seed, ws.ptr, _stream(stream)), "nvfp4_amax")
    return ws


def nvfp4_quantize_dual_shard(x: torch.Tensor, row_offset: int, rows_total: int, mode: int = RNE, rht_seed: int = 0,
                              sr_seed: int = 0, stream_row: int = 0, stream_col: int = 0,
                              out_row: NVFP4Tensor | None = None, out_col: NVFP4Tensor | None = None,
                              ws: Workspace | None = None, stream=None):
    """Pass 2 of nvfp4_quantize_dual for rows [row_offset, row_offset + rows) of a rows_total-row
    tensor, with the (reduced) amax words already in ws."""
    rows, cols, ld = _bf16_2d(x)
    out_row = out_row or NVFP4Tensor.empty(rows, cols, BLOCK_1x16, x.device)
    out_col = out_col or NVFP4Tensor.empty(cols, rows, BLOCK_1x16, x.device)
    ws = ws or default_workspace()
    a, b = out_row.c(), out_col.c()
    st = _lib().nvfp4_quantize_dual_shard(_ptr(x), rows, cols, ld, row_offset, rows_total, mode, rht_seed, sr_seed,
                                          stream_row, stream_col, ctypes.byref(a), ctypes.byref(b), ws.ptr,
                                          _stream(stream))
    _check(st, "nvfp4_quantize_dual_shard")
    return out_row, out_col


def nvfp4_quantize_dual_dp(x: torch.Tensor, group, row_offset: int, rows_total: int, mode: int = RNE,
                           rht_seed: int = 0, sr_seed: int = 0, stream_row: int = 0, stream_col: int = 0,
                           out_row: NVFP4Tensor | None = None, out_col: NVFP4Tensor | None = None,
                           ws: Workspace | None = None, stream=None):
    """Both forms of this rank's token shard, equal to the slices of the whole batch's forms: the
    shard amax, a MAX all-reduce of the two amax words over ``group`` (torch.distributed), then
    the shard's pass 2.  Without an initialized process group there is one rank, whose shard is
    the batch, and no exchange."""
    import torch.distributed as dist
    ws = nvfp4_amax(x, True, rht_seed, ws, stream)
    if dist.is_initialized():
        dist.all_reduce(ws.amax_words(), op=dist.ReduceOp.MAX, group=group)
    return nvfp4_quantize_dual_shard(x, row_offset, rows_total, mode, rht_seed, sr_seed, stream_row, stream_col,
                                     out_row, out_col, ws, stream)


def nvfp4_quantize_weight(w: torch.Tensor, transposed: bool = True, out: NVFP4Tensor | None = None,
                          out_t: NVFP4Tensor | None = None, ws: Workspace | None = None, stream=None):
    rows, cols, ld = _bf16_2d(w)
    out = out or NVFP4Tensor.empty(rows, cols, BLOCK_16x16, w.device)
    if transposed:
        out_t = out_t or NVFP4Tensor.empty(cols, rows, BLOCK_16x16, w.device)
    ws = ws or default_workspace()
    a = out.c()
    b = out_t.c() if transposed else None
    st = _lib().nvfp4_quantize_weight(_ptr(w), rows, cols, ld, ctypes.byref(a), ctypes.byref(b) if b else None,
                                      ws.ptr, _stream(stream))
    _check(st, "nvfp4_quantize_weight")
    return (out, out_t) if transposed else out


def nvfp4_transpose_2d(w: NVFP4Tensor, out: NVFP4Tensor | None = None, stream=None) -> NVFP4Tensor:
    out = out or NVFP4Tensor.empty(w.k, w.rows, BLOCK_16x16, w.codes.device)
    a, b = w.c(), out.c()
    _check(_lib().nvfp4_transpose_2d(ctypes.byref(a), ctypes.byref(b), _stream(stream)), "nvfp4_transpose_2d")
    return out


def nvfp4_gemm(a: NVFP4Tensor, b: NVFP4Tensor, out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
               ws: Workspace | None = None, stream=None) -> torch.Tensor:
    """D[M][N] = s_tA s_tB * A . B^T (both K-major quantized forms)."""
    M, N = a.rows, b.rows
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=a.codes.device)
    code = OUT_FP32 if out.dtype == torch.float32 else OUT_BF16
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("output must be bf16 or fp32")
    ws = ws or default_workspace()
    ca, cb = a.c(), b.c()
    st = _lib().nvfp4_gemm(ctypes.byref(ca), ctypes.byref(cb), _ptr(out), out.stride(0), code, ws.ptr, _stream(stream))
    _check(st, "nvfp4_gemm")
    return out


def nvfp4_gemm_amax(a: NVFP4Tensor, b: NVFP4Tensor, amax_ws: Workspace, rht_seed: int = 0,
                    out: torch.Tensor | None = None, ws: Workspace | None = None, stream=None) -> torch.Tensor:
    """D = s_tA s_tB * A . B^T in bf16, with D's plain and RHT amax written into amax_ws (as
    nvfp4_amax(D, True, rht_seed, amax_ws) would), ready for the quantize call that reads D."""
    M, N = a.rows, b.rows
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a.codes.device)
    if out.dtype != torch.bfloat16:
        raise TypeError("nvfp4_gemm_amax writes bf16")
    ws = ws or default_workspace()
    ca, cb = a.c(), b.c()
    st = _lib().nvfp4_gemm_amax(ctypes.byref(ca), ctypes.byref(cb), _ptr(out), out.stride(0), rht_seed, amax_ws.ptr,
                                ws.ptr, _stream(stream))
    _check(st, "nvfp4_gemm_amax")
    return out


def nvfp4_gemm_reduce_scatter(a: NVFP4Tensor, b: NVFP4Tensor, shards, owner_rows: int,
                              ws: Workspace | None = None, stream=None) -> None:
    """shards[o] += rows [o*owner_rows, (o+1)*owner_rows) of s_tA s_tB * A . B^T (fp32 adds).

    shards: fp32 [rows_o][N] tensors with one row stride (local, or another GPU's buffer through
    a peer mapping). One owner with owner_rows >= rows accumulates the whole product into it.
    """
    if not shards:
        raise ValueError("nvfp4_gemm_reduce_scatter needs at least one shard")
    ld = shards[0].stride(0)
    for t in shards:
        if t.dtype != torch.float32 or t.dim() != 2 or t.stride(1) != 1 or t.stride(0) != ld:
            raise ValueError("shards must be fp32 2-D row-major tensors with one row stride")
        if t.shape[1] != b.rows:
            raise ValueError("each shard has N = b.rows columns")
    for o, t in enumerate(shards):
        if t.shape[0] < min(owner_rows, a.rows - o * owner_rows):
            raise ValueError(f"shard {o} holds fewer rows than its owner's share")
    addrs = (ctypes.c_void_p * len(shards))(*[t.data_ptr() for t in shards])
    ws = ws or default_workspace()
    ca, cb = a.c(), b.c()
    st = _lib().nvfp4_gemm_reduce_scatter(ctypes.byref(ca), ctypes.byref(cb), addrs, len(shards), owner_rows, ld,
                                          ws.ptr, _stream(stream))
    _check(st, "nvfp4_gemm_reduce_scatter")


def nvfp4_gelu_fwd(h: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    out = torch.empty_like(h) if out is None else out
    _check(_lib().nvfp4_gelu_fwd(_ptr(h), _ptr(out), h.numel(), _stream(stream)), "nvfp4_gelu_fwd")
    return out


def nvfp4_gelu_bwd(h: torch.Tensor, dg: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    out = torch.empty_like(h) if out is None else out
    _check(_lib().nvfp4_gelu_bwd(_ptr(h), _ptr(dg), _ptr(out), h.numel(), _stream(stream)), "nvfp4_gelu_bwd")
    return out


def nvfp4_gelu_fwd_amax(h: torch.Tensor, out: torch.Tensor | None = None, rht_seed: int = 0,
                        ws: Workspace | None = None, stream=None) -> torch.Tensor:
    """GeLU of h [rows][cols] with the plain and RHT amax of the bf16 result into ws."""
    rows, cols, ld = _bf16_2d(h)
    if ld != cols:
        raise ValueError("nvfp4_gelu_fwd_amax needs a contiguous input")
    out = torch.empty_like(h) if out is None else out
    ws = ws or default_workspace()
    _check(_lib().nvfp4_gelu_fwd_amax(_ptr(h), _ptr(out), rows, cols, rht_seed, ws.ptr, _stream(stream)),
           "nvfp4_gelu_fwd_amax")
    return out


def nvfp4_gelu_bwd_amax(h: torch.Tensor, dg: torch.Tensor, out: torch.Tensor | None = None, rht_seed: int = 0,
                        ws: Workspace | None = None, stream=None) -> torch.Tensor:
    """dg * GeLU'(h) with the plain and RHT amax of the bf16 result into ws."""
    rows, cols, ld = _bf16_2d(h)
    if ld != cols or not dg.is_contiguous():
        raise ValueError("nvfp4_gelu_bwd_amax needs contiguous inputs")
    out = torch.empty_like(h) if out is None else out
    ws = ws or default_workspace()
    _check(_lib().nvfp4_gelu_bwd_amax(_ptr(h), _ptr(dg), _ptr(out), rows, cols, rht_seed, ws.ptr, _stream(stream)),
           "nvfp4_gelu_bwd_amax")
    return out


# ---------------------------------------------------------------------------------------
# MXFP4 (the comparison format: blocks of 32, UE8M0 scales, no tensor scale)
# ---------------------------------------------------------------------------------------
@dataclass
class MXTensor:
    """One MXFP4 operand form (device buffers owned by torch)."""
    codes: torch.Tensor          # uint8 [rows][k/2]
    scales: torch.Tensor         # uint8, 128x4-tile swizzled UE8M0 block scales
    rows: int
    k: int

    @staticmethod
    def empty(rows: int, k: int, device=None) -> "MXTensor":
        L = _lib()
        device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        codes = torch.empty(max(L.nvfp4_codes_bytes(rows, k), 1), dtype=torch.uint8, device=device)
        scales = torch.empty(max(L.nvfp4_mx_scales_bytes(rows, k), 16), dtype=torch.uint8, device=device)
        return MXTensor(codes, scales, rows, k)

    def c(self) -> CMXTensor:
        return CMXTensor(self.codes.data_ptr(), self.scales.data_ptr(), self.rows, self.k)


def nvfp4_mx_quantize(x: torch.Tensor, along: int = 0, mode: int = RNE, sr_seed: int = 0, stream_id: int = 0,
                      out: MXTensor | None = None, ws: Workspace | None = None, stream=None) -> MXTensor:
    rows, cols, ld = _bf16_2d(x)
    R, K = (cols, rows) if along else (rows, cols)
    out = out or MXTensor.empty(R, K, x.device)
    ws = ws or default_workspace()
    ct = out.c()
    _check(_lib().nvfp4_mx_quantize(_ptr(x), rows, cols, ld, along, mode, sr_seed, stream_id, ctypes.byref(ct), ws.ptr,
                                    _stream(stream)), "nvfp4_mx_quantize")
    return out


def nvfp4_mx_quantize_dual(x: torch.Tensor, mode: int = RNE, sr_seed: int = 0, stream_row: int = 0, stream_col: int = 0,
                           out_row: MXTensor | None = None, out_col: MXTensor | None = None,
                           ws: Workspace | None = None, stream=None):
    """Both MXFP4 forms of x (along 0 and along 1) from one read."""
    rows, cols, ld = _bf16_2d(x)
    out_row = out_row or MXTensor.empty(rows, cols, x.device)
    out_col = out_col or MXTensor.empty(cols, rows, x.device)
    ws = ws or default_workspace()
    a, b = out_row.c(), out_col.c()
    _check(_lib().nvfp4_mx_quantize_dual(_ptr(x), rows, cols, ld, mode, sr_seed, stream_row, stream_col,
                                         ctypes.byref(a), ctypes.byref(b), ws.ptr, _stream(stream)),
           "nvfp4_mx_quantize_dual")
    return out_row, out_col


def nvfp4_mx_gemm(a: MXTensor, b: MXTensor, out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
                  ws: Workspace | None = None, stream=None) -> torch.Tensor:
    """D[M][N] = A . B^T over MXFP4 forms (kind::mxf4 block-scaled MMA)."""
    if out is None:
        out = torch.empty((a.rows, b.rows), dtype=out_dtype, device=a.codes.device)
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("output must be bf16 or fp32")
    code = OUT_FP32 if out.dtype == torch.float32 else OUT_BF16
    ws = ws or default_workspace()
    ca, cb = a.c(), b.c()
    _check(_lib().nvfp4_mx_gemm(ctypes.byref(ca), ctypes.byref(cb), _ptr(out), out.stride(0), code, ws.ptr,
                                _stream(stream)), "nvfp4_mx_gemm")
    return out


# ---------------------------------------------------------------------------------------
# BF16 path (the layers kept in high precision)
# ---------------------------------------------------------------------------------------
def nvfp4_bf16_gemm(a: torch.Tensor, b: torch.Tensor, out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
                    ws: Workspace | None = None, stream=None) -> torch.Tensor:
    """D[M][N] = A[M][K] . B[N][K]^T for bf16 A, B (tcgen05 kind::f16, fp32 accumulation)."""
    M, K, lda = _bf16_2d(a)
    N, Kb, ldb = _bf16_2d(b)
    if Kb != K:
        raise ValueError("A and B need the same K")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=a.device)
    code = OUT_FP32 if out.dtype == torch.float32 else OUT_BF16
    ws = ws or default_workspace()
    _check(_lib().nvfp4_bf16_gemm(_ptr(a), lda, _ptr(b), ldb, M, N, K, _ptr(out), out.stride(0), code, ws.ptr,
                                  _stream(stream)), "nvfp4_bf16_gemm")
    return out


def nvfp4_bf16_transpose(x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    rows, cols, ld = _bf16_2d(x)
    out = torch.empty((cols, rows), dtype=torch.bfloat16, device=x.device) if out is None else out
    _check(_lib().nvfp4_bf16_transpose(_ptr(x), rows, cols, ld, _ptr(out), out.stride(0), _stream(stream)),
           "nvfp4_bf16_transpose")
    return out


class LinearBF16:
    """The BF16 linear layer y = x w^T with its caller-owned transpose scratch."""

    def __init__(self, T: int, d: int, n: int, device=None):
        device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        self.T, self.d, self.n = T, d, n
        self.scratch = torch.empty(max(_lib().nvfp4_linear_bf16_scratch_bytes(T, d, n), 16), dtype=torch.uint8,
                                   device=device)
        self.ws = Workspace(device)

    def fwd(self, x: torch.Tensor, w: torch.Tensor, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        y = torch.empty((self.T, self.n), dtype=torch.bfloat16, device=x.device) if y is None else y
        _check(_lib().nvfp4_linear_bf16_fwd(_ptr(x), _ptr(w), _ptr(y), self.T, self.d, self.n, self.ws.ptr,
                                            _stream(stream)), "nvfp4_linear_bf16_fwd")
        return y

    def bwd(self, x: torch.Tensor, w: torch.Tensor, dy: torch.Tensor, dx: torch.Tensor | None = None,
            dw: torch.Tensor | None = None, stream=None):
        dx = torch.empty((self.T, self.d), dtype=torch.bfloat16, device=x.device) if dx is None else dx
        dw = torch.empty((self.n, self.d), dtype=torch.float32, device=x.device) if dw is None else dw
        _check(_lib().nvfp4_linear_bf16_bwd(_ptr(x), _ptr(w), _ptr(dy), _ptr(dx), _ptr(dw), self.T, self.d, self.n,
                                            _ptr(self.scratch), self.ws.ptr, _stream(stream)), "nvfp4_linear_bf16_bwd")
        return dx, dw


# ---------------------------------------------------------------------------------------
# linear layer
# ---------------------------------------------------------------------------------------
class LinearContext:
    """Caller-owned buffers of one NVFP4 linear layer y = x w^T (T tokens, d in, n out)."""

    def __init__(self, T: int, d: int, n: int, rht_seed: int = 0, device=None):
        device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        self.T, self.d, self.n = T, d, n
        self.xq = NVFP4Tensor.empty(T, d, BLOCK_1x16, device)
        self.xq_rht = NVFP4Tensor.empty(d, T, BLOCK_1x16, device)
        self.wq = NVFP4Tensor.empty(n, d, BLOCK_16x16, device)
        self.wqt = NVFP4Tensor.empty(d, n, BLOCK_16x16, device)
        self.dyq = NVFP4Tensor.empty(T, n, BLOCK_1x16, device)
        self.dyq_rht = NVFP4Tensor.empty(n, T, BLOCK_1x16, device)
        self.ws = Workspace(device)
        self.ctx = CLinearCtx(T, d, n, rht_seed, self.xq.c(), self.xq_rht.c(), self.wq.c(), self.wqt.c(),
                              self.dyq.c(), self.dyq_rht.c(), self.ws.buf.data_ptr(), 0, 0)

    @property
    def w_cached(self) -> bool:
        return bool(self.ctx.w_cached)

    @w_cached.setter
    def w_cached(self, v: bool):
        self.ctx.w_cached = 1 if v else 0

    @property
    def amax_ready(self) -> bool:
        """The next call's input has its amax words in this context's workspace already (a fused
        producer wrote them); the call skips its amax pass and clears the flag."""
        return bool(self.ctx.amax_ready)

    @amax_ready.setter
    def amax_ready(self, v: bool):
        self.ctx.amax_ready = 1 if v else 0

    def feed(self, consumer: "LinearContext"):
        """This layer's y is consumer's x and consumer's dx is this layer's dy (a stack of layers):
        this layer's fprop GEMM writes y's amax words into consumer's workspace, and consumer's
        dgrad GEMM writes dx's into this layer's, so the consuming quantize calls skip their amax
        passes (the caller sets amax_ready on the consuming context before its call)."""
        self.ctx.y_amax_ws = consumer.ws.ptr
        self.ctx.y_rht_seed = consumer.ctx.rht_seed
        consumer.ctx.dx_amax_ws = self.ws.ptr
        consumer.ctx.dx_rht_seed = self.ctx.rht_seed
        # each context now holds the other's workspace address: keep both workspaces alive
        self._feeds = consumer
        consumer._fed_by = self


# ---------------------------------------------------------------------------------------
# data parallelism over tokens
# ---------------------------------------------------------------------------------------
def dp_token_rows(T_local: int, rank: int, world: int):
    """(row_offset, rows_total) of this rank's token shard in the whole batch: ranks hold equal
    consecutive shards in rank order."""
    return rank * T_local, world * T_local


def dp_dw_rows(n: int, rank: int, world: int):
    """The rows [r0, r1) of dW that the reduce-scatter leaves on this rank (n % world == 0)."""
    if n % world:
        raise ValueError("out-features must divide evenly over the ranks")
    per = n // world
    return rank * per, (rank + 1) * per


class DPLinear:
    """The NVFP4 linear layer y = x w^T under data parallelism: each rank holds T consecutive tokens
    of a world * T-token batch and a replica of w.

    - X and dY: the tensor scale comes from the whole batch, so the plain and RHT amax of each
      rank's shard are all-reduced with an integer MAX between the two quantize passes, and SR
      fields are indexed in the whole batch's forms: every rank's forms are its slice of the forms
      one GPU would compute for the whole batch.
    - W: quantized on every rank from the same replica (identical forms, no exchange).
    - dW: each rank's wgrad GEMM gives the partial sum over its tokens; the partials are
      reduce-scattered (fp32 sum) over the group, each rank keeping rows dp_dw_rows(n, rank,
      world).  dw_reduce="nccl": the wgrad GEMM stores the partial, and an NCCL reduce-scatter
      overlaps the dgrad GEMM.  dw_reduce="fused": the wgrad GEMM's epilogue adds each output
      tile into its owner's shard directly (nvfp4_gemm_reduce_scatter into the ranks' symmetric
      buffers, through peer addresses), so the exchange runs inside the GEMM; a 4-byte all-reduce
      after the dgrad GEMM is the barrier that orders every rank's adds before the owner reads
      its shard.  Two shard buffers alternate between steps, so a buffer is zeroed one whole
      step (one barrier) before any rank adds into it again.
    """

    def __init__(self, T: int, d: int, n: int, group=None, rht_seed: int = 0, device=None,
                 dw_reduce: str = "nccl"):
        import torch.distributed as dist
        if dw_reduce not in ("nccl", "fused"):
            raise ValueError("dw_reduce is 'nccl' or 'fused'")
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        self.T, self.d, self.n, self.rht_seed = T, d, n, rht_seed
        self.ctx = LinearContext(T, d, n, rht_seed=rht_seed, device=device)
        r0, r1 = dp_dw_rows(n, self.rank, self.world)
        self.dw = torch.empty((r1 - r0, d), dtype=torch.float32, device=device)
        self.dw_reduce = dw_reduce
        if dw_reduce == "nccl":
            self.dw_partial = torch.empty((n, d), dtype=torch.float32, device=device)
            return
        per = r1 - r0
        if per % 32 or self.world > 8:
            raise ValueError("the fused reduce-scatter needs n / world % 32 == 0 and at most 8 ranks")
        self._rs_bufs, self._rs_peers, self._rs_step = [], [], 0
        for _ in range(2):
            if dist.is_initialized():
                import torch.distributed._symmetric_memory as symm_mem
                buf = symm_mem.empty((per, d), dtype=torch.float32, device=device)
                buf.zero_()
                h = symm_mem.rendezvous(buf, group if group is not None else dist.group.WORLD)
                peers = [buf if p == self.rank else h.get_buffer(p, (per, d), torch.float32)
                         for p in range(self.world)]
            else:
                buf = torch.zeros((per, d), dtype=torch.float32, device=device)
                peers = [buf]
            self._rs_bufs.append(buf)
            self._rs_peers.append(peers)
        self._rs_flag = torch.zeros(1, dtype=torch.float32, device=device)
        if dist.is_initialized():
            torch.cuda.synchronize(device)
            dist.barrier(group)   # every shard is zero before any rank adds into it

    def fwd(self, x: torch.Tensor, w: torch.Tensor, y: torch.Tensor | None = None) -> torch.Tensor:
        c = self.ctx
        off, total = dp_token_rows(self.T, self.rank, self.world)
        nvfp4_quantize_dual_dp(x, self.group, off, total, mode=RNE, rht_seed=self.rht_seed, out_row=c.xq,
                               out_col=c.xq_rht, ws=c.ws)
        nvfp4_quantize_weight(w, out=c.wq, out_t=c.wqt, ws=c.ws)
        return nvfp4_gemm(c.xq, c.wq, out=y, ws=c.ws)

    def bwd(self, dy: torch.Tensor, sr_seed: int, dx: torch.Tensor | None = None):
        """dX for this rank's tokens; this rank's rows of the batch's dW land in self.dw."""
        import torch.distributed as dist
        c = self.ctx
        off, total = dp_token_rows(self.T, self.rank, self.world)
        nvfp4_quantize_dual_dp(dy, self.group, off, total, mode=SR, rht_seed=self.rht_seed, sr_seed=sr_seed,
                               stream_row=STREAM_DGRAD, stream_col=STREAM_WGRAD, out_row=c.dyq, out_col=c.dyq_rht,
                               ws=c.ws)
        if self.dw_reduce == "fused":
            j = self._rs_step & 1
            self._rs_step += 1
            nvfp4_gemm_reduce_scatter(c.dyq_rht, c.xq_rht, self._rs_peers[j], self.dw.shape[0], ws=c.ws)
            dx = nvfp4_gemm(c.dyq, c.wqt, out=dx, ws=c.ws)
            if dist.is_initialized():
                dist.all_reduce(self._rs_flag, group=self.group)   # every rank's adds are complete
            self.dw.copy_(self._rs_bufs[j])
            self._rs_bufs[j].zero_()
            return dx
        nvfp4_gemm(c.dyq_rht, c.xq_rht, out=self.dw_partial, ws=c.ws)
        work = None
        if self.world > 1:
            work = dist.reduce_scatter_tensor(self.dw, self.dw_partial, op=dist.ReduceOp.SUM, group=self.group,
                                              async_op=True)
        dx = nvfp4_gemm(c.dyq, c.wqt, out=dx, ws=c.ws)
        if work is not None:
            work.wait()
        else:
            self.dw.copy_(self.dw_partial)
        return dx


def nvfp4_linear_fwd(ctx: LinearContext, x: torch.Tensor, w: torch.Tensor | None, y: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    if y is None:
        y = torch.empty((ctx.T, ctx.n), dtype=torch.bfloat16, device=x.device)
    st = _lib().nvfp4_linear_fwd(_ptr(x), _ptr(w), _ptr(y), ctypes.byref(ctx.ctx), _stream(stream))
    _check(st, "nvfp4_linear_fwd")
    return y


def nvfp4_linear_bwd(ctx: LinearContext, dy: torch.Tensor, sr_seed: int, dx: torch.Tensor | None = None,
                     dw: torch.Tensor | None = None, stream=None):
    if dx is None:
        dx = torch.empty((ctx.T, ctx.d), dtype=torch.bfloat16, device=dy.device)
    if dw is None:
        dw = torch.empty((ctx.n, ctx.d), dtype=torch.float32, device=dy.device)
    st = _lib().nvfp4_linear_bwd(_ptr(dy), sr_seed, _ptr(dx), _ptr(dw), ctypes.byref(ctx.ctx), _stream(stream))
    _check(st, "nvfp4_linear_bwd")
    return dx, dw
