"""CPU oracle for the NVFP4 linear-layer hot path -- TEST INFRASTRUCTURE ONLY.

Thin ctypes/numpy wrapper around ``nvfp4_oracle.c`` (plain scalar C, fp32 steps in the pages'
order, fp64 GEMM).  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline / reference arm may import this package.  It imports nothing from the CUDA package
and the CUDA package imports nothing from here.

Parity status of each function (pins live in ``tests/test_oracle_*.py``):
- E2M1 / E4M3 encode and decode: pinned against ``ml_dtypes`` (exhaustive on the decision
  ranges) and hand-worked values under ``tests/golden``.
- Philox4x32-10: pinned on CPU only statistically; pinned exactly on the GPU against cuRAND's
  independent Philox4_32_10 generator (``tests/test_gpu_encoders.py``).
- RHT butterfly: pinned against the closed-form Sylvester matrix in fp64, orthogonality and
  the exact one-hot response.
- SR: pinned by unbiasedness and frequency statistics at 3 sigma over 1e6 draws.
- Quantizers: pinned by the 6.25 % invariant, the reconstruction bound, the transpose identity
  of 16x16 blocks and a hand-worked block.
- GEMM: pinned against numpy matmul of operands decoded through ``ml_dtypes``.
- GeLU glue: pinned against scipy's normal CDF, closed forms and finite differences.
- MXFP4 quantizer (the pages' comparison format): pinned against an encoder built from
  ``ml_dtypes`` (E2M1 and E8M0) and numpy's frexp, the scale's closed form per binade and
  the reconstruction bound (``tests/test_oracle_mx.py``).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None

RNE, SR = 0, 1
BLOCK_1x16, BLOCK_16x16 = 0, 1
OK, ERR_SHAPE, ERR_NONFINITE, ERR_ARG, ERR_NOMEM = 0, 1, 2, 3, 4


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        c = ctypes
        u8p, u16p, u32p, u64p = (c.POINTER(c.c_uint8), c.POINTER(c.c_uint16),
                                 c.POINTER(c.c_uint32), c.POINTER(c.c_uint64))
        f32p, f64p, i64p = c.POINTER(c.c_float), c.POINTER(c.c_double), c.POINTER(c.c_int64)
        L.ora_bf16_to_f32.argtypes = [c.c_uint16]; L.ora_bf16_to_f32.restype = c.c_float
        L.ora_f32_to_bf16.argtypes = [c.c_float]; L.ora_f32_to_bf16.restype = c.c_uint16
        L.ora_e2m1_value.argtypes = [c.c_uint8]; L.ora_e2m1_value.restype = c.c_double
        L.ora_e2m1_rne.argtypes = [c.c_float]; L.ora_e2m1_rne.restype = c.c_uint8
        L.ora_e2m1_sr.argtypes = [c.c_float, c.c_uint32]; L.ora_e2m1_sr.restype = c.c_uint8
        L.ora_e4m3_value.argtypes = [c.c_uint8]; L.ora_e4m3_value.restype = c.c_double
        L.ora_e4m3_rne_sat.argtypes = [c.c_float]; L.ora_e4m3_rne_sat.restype = c.c_uint8
        L.ora_philox4x32_10.argtypes = [u32p, u32p, u32p]; L.ora_philox4x32_10.restype = None
        L.ora_sr_bits16.argtypes = [c.c_uint64, c.c_uint32, c.c_uint64]; L.ora_sr_bits16.restype = c.c_uint32
        L.ora_rht_signs.argtypes = [c.c_uint64]; L.ora_rht_signs.restype = c.c_uint32
        L.ora_rht16.argtypes = [f32p, c.c_uint32]; L.ora_rht16.restype = None
        L.ora_swizzle_offset.argtypes = [c.c_int64, c.c_int64, c.c_int64]; L.ora_swizzle_offset.restype = c.c_int64
        L.ora_scales_sw_bytes.argtypes = [c.c_int64, c.c_int64]; L.ora_scales_sw_bytes.restype = c.c_int64
        L.ora_quantize.argtypes = [u16p, c.c_int64, c.c_int64, c.c_int64, c.c_int, c.c_int, c.c_int, c.c_int,
                                   c.c_uint64, c.c_uint64, c.c_uint32, u8p, u8p, u8p, u8p, f32p, f32p, c.c_int]
        L.ora_quantize.restype = c.c_int
        L.ora_transpose_2d.argtypes = [u8p, u8p, c.c_int64, c.c_int64, u8p, u8p, u8p, u8p]
        L.ora_transpose_2d.restype = c.c_int
        L.ora_dequantize.argtypes = [u8p, u8p, c.c_float, c.c_int64, c.c_int64, f64p]
        L.ora_dequantize.restype = None
        L.ora_gemm_sampled.argtypes = [u8p, u8p, c.c_float, u8p, u8p, c.c_float, c.c_int64,
                                       i64p, i64p, c.c_int64, f64p, f64p, c.c_int]
        L.ora_gemm_sampled.restype = c.c_int
        L.ora_gemm_full.argtypes = [u8p, u8p, c.c_float, u8p, u8p, c.c_float, c.c_int64, c.c_int64, c.c_int64,
                                    f64p, f64p]
        L.ora_gemm_full.restype = c.c_int
        L.ora_gelu_fwd.argtypes = [u16p, c.c_int64, u16p]; L.ora_gelu_fwd.restype = None
        L.ora_gelu_bwd.argtypes = [u16p, u16p, c.c_int64, u16p]; L.ora_gelu_bwd.restype = None
        L.ora_e2m1_rne_batch.argtypes = [f32p, c.c_int64, u8p]; L.ora_e2m1_rne_batch.restype = None
        L.ora_e2m1_sr_batch.argtypes = [f32p, u32p, c.c_int64, u8p]; L.ora_e2m1_sr_batch.restype = None
        L.ora_e2m1_sr_threshold_batch.argtypes = [f32p, c.c_int64, u32p]
        L.ora_e2m1_sr_threshold_batch.restype = None
        L.ora_e4m3_rne_sat_batch.argtypes = [f32p, c.c_int64, u8p]; L.ora_e4m3_rne_sat_batch.restype = None
        L.ora_sr_bits16_batch.argtypes = [c.c_uint64, c.c_uint32, u64p, c.c_int64, u32p]
        L.ora_sr_bits16_batch.restype = None
        L.ora_philox_batch.argtypes = [c.c_uint64, c.c_uint32, c.c_uint64, c.c_int64, u32p]
        L.ora_philox_batch.restype = None
        L.ora_ue8m0_of_amax.argtypes = [c.c_float]
        L.ora_ue8m0_of_amax.restype = c.c_uint8
        L.ora_quantize_mx.argtypes = [u16p, c.c_int64, c.c_int64, c.c_int64, c.c_int, c.c_uint64, c.c_uint32, u8p, u8p]
        L.ora_quantize_mx.restype = c.c_int
        L.ora_dequantize_mx.argtypes = [u8p, u8p, c.c_int64, c.c_int64, f64p]
        L.ora_dequantize_mx.restype = None
        L.ora_mx_scales_swizzle.argtypes = [u8p, c.c_int64, c.c_int64, u8p]
        L.ora_mx_scales_swizzle.restype = None
        _LIB = L
    return _LIB


def _p(a: np.ndarray, ctype):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _p_or_null(a, ctype):
    return ctypes.POINTER(ctype)() if a is None else _p(a, ctype)


def default_threads() -> int:
    return os.cpu_count() or 1


# ---------------------------------------------------------------------------------------
# element-level helpers
# ---------------------------------------------------------------------------------------
def e2m1_rne(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().ora_e2m1_rne_batch(_p(x, ctypes.c_float), x.size, _p(out, ctypes.c_uint8))
    return out


def e2m1_sr(x: np.ndarray, r16: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    r16 = np.ascontiguousarray(r16, dtype=np.uint32)
    out = np.empty(x.shape, np.uint8)
    lib().ora_e2m1_sr_batch(_p(x, ctypes.c_float), _p(r16, ctypes.c_uint32), x.size, _p(out, ctypes.c_uint8))
    return out


def e2m1_sr_threshold(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint32)
    lib().ora_e2m1_sr_threshold_batch(_p(x, ctypes.c_float), x.size, _p(out, ctypes.c_uint32))
    return out


def e4m3_rne_sat(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().ora_e4m3_rne_sat_batch(_p(x, ctypes.c_float), x.size, _p(out, ctypes.c_uint8))
    return out


def e2m1_value(code: int) -> float:
    return lib().ora_e2m1_value(code)


def e4m3_value(code: int) -> float:
    return lib().ora_e4m3_value(code)


def philox4x32_10(ctr, key):
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.empty(4, np.uint32)
    lib().ora_philox4x32_10(_p(c, ctypes.c_uint32), _p(k, ctypes.c_uint32), _p(out, ctypes.c_uint32))
    return out


def philox_blocks(seed: int, stream_id: int, g0: int, n: int) -> np.ndarray:
    out = np.empty((n, 4), np.uint32)
    lib().ora_philox_batch(seed, stream_id, g0, n, _p(out, ctypes.c_uint32))
    return out


def sr_bits16(seed: int, stream_id: int, idx: np.ndarray) -> np.ndarray:
    idx = np.ascontiguousarray(idx, dtype=np.uint64)
    out = np.empty(idx.shape, np.uint32)
    lib().ora_sr_bits16_batch(seed, stream_id, _p(idx, ctypes.c_uint64), idx.size, _p(out, ctypes.c_uint32))
    return out


def rht_signs(seed: int) -> int:
    return lib().ora_rht_signs(seed)


def rht16(v: np.ndarray, signs: int) -> np.ndarray:
    a = np.array(v, dtype=np.float32, copy=True).reshape(16)
    lib().ora_rht16(_p(a, ctypes.c_float), signs)
    return a


def swizzle_offset(r: int, kb: int, K: int) -> int:
    return lib().ora_swizzle_offset(r, kb, K)


def scales_sw_bytes(R: int, K: int) -> int:
    return lib().ora_scales_sw_bytes(R, K)


# ---------------------------------------------------------------------------------------
# operand forms
# ---------------------------------------------------------------------------------------
class QForm:
    """One quantized operand form: R rows, K along the GEMM reduction axis."""

    def __init__(self, R, K, codes, scales_rm, scales_sw, tile_scales, amax, s_t):
        self.R, self.K = R, K
        self.codes = codes            # uint8 [R][K/2], even k in the low nibble
        self.scales_rm = scales_rm    # uint8 [R][K/16]
        self.scales_sw = scales_sw    # uint8, 128x4 tiles
        self.tile_scales = tile_scales
        self.amax = amax
        self.s_t = s_t

    def nibbles(self) -> np.ndarray:
        lo = self.codes & 15
        hi = self.codes >> 4
        out = np.empty((self.R, self.K), np.uint8)
        out[:, 0::2] = lo
        out[:, 1::2] = hi
        return out

    def dequantize(self) -> np.ndarray:
        out = np.empty((self.R, self.K), np.float64)
        lib().ora_dequantize(_p(self.codes, ctypes.c_uint8), _p(self.scales_rm, ctypes.c_uint8),
                             self.s_t, self.R, self.K, _p(out, ctypes.c_double))
        return out


def quantize(x_bits: np.ndarray, along: int = 0, mode: int = RNE, block: int = BLOCK_1x16, rht: bool = False,
             rht_seed: int = 0, sr_seed: int = 0, stream_id: int = 0, nthreads: int | None = None,
             ld: int | None = None) -> QForm:
    """Quantize a bf16 tensor given as its uint16 bit patterns, shape [rows][cols]."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    rows, cols = x_bits.shape
    if ld is None:
        ld = cols
    R, K = (cols, rows) if along else (rows, cols)
    codes = np.zeros((R, K // 2), np.uint8)
    scales_rm = np.zeros((R, max(K // 16, 0)), np.uint8)
    scales_sw = np.zeros(max(scales_sw_bytes(R, K), 0), np.uint8)
    tile = np.zeros((R // 16, K // 16), np.uint8) if block == BLOCK_16x16 else None
    amax = ctypes.c_float(0)
    s_t = ctypes.c_float(0)
    st = lib().ora_quantize(_p(x_bits, ctypes.c_uint16), rows, cols, ld, along, mode, block, int(rht),
                            rht_seed, sr_seed, stream_id, _p(codes, ctypes.c_uint8), _p(scales_rm, ctypes.c_uint8),
                            _p(scales_sw, ctypes.c_uint8), _p_or_null(tile, ctypes.c_uint8), ctypes.byref(amax),
                            ctypes.byref(s_t), nthreads or default_threads())
    if st != OK:
        raise ValueError(f"oracle quantize failed with status {st}")
    return QForm(R, K, codes, scales_rm, scales_sw, tile, amax.value, s_t.value)


def transpose_2d(q: QForm) -> QForm:
    R, K = q.R, q.K
    codes_t = np.zeros((K, R // 2), np.uint8)
    scales_rm_t = np.zeros((K, R // 16), np.uint8)
    scales_sw_t = np.zeros(scales_sw_bytes(K, R), np.uint8)
    tile_t = np.zeros((K // 16, R // 16), np.uint8)
    st = lib().ora_transpose_2d(_p(q.codes, ctypes.c_uint8), _p(q.tile_scales, ctypes.c_uint8), R, K,
                                _p(codes_t, ctypes.c_uint8), _p(scales_rm_t, ctypes.c_uint8),
                                _p(scales_sw_t, ctypes.c_uint8), _p(tile_t, ctypes.c_uint8))
    if st != OK:
        raise ValueError(f"oracle transpose failed with status {st}")
    return QForm(K, R, codes_t, scales_rm_t, scales_sw_t, tile_t, q.amax, q.s_t)


def gemm_full(a: QForm, b: QForm):
    """D = A * B^T in fp64 over the dequantized forms, plus sum_k |a_ik b_jk|."""
    assert a.K == b.K
    d = np.empty((a.R, b.R), np.float64)
    s = np.empty((a.R, b.R), np.float64)
    st = lib().ora_gemm_full(_p(a.codes, ctypes.c_uint8), _p(a.scales_rm, ctypes.c_uint8), a.s_t,
                             _p(b.codes, ctypes.c_uint8), _p(b.scales_rm, ctypes.c_uint8), b.s_t,
                             a.R, b.R, a.K, _p(d, ctypes.c_double), _p(s, ctypes.c_double))
    if st != OK:
        raise ValueError(f"oracle gemm failed with status {st}")
    return d, s


def gemm_sampled(a: QForm, b: QForm, ii: np.ndarray, jj: np.ndarray, nthreads: int | None = None):
    assert a.K == b.K
    ii = np.ascontiguousarray(ii, dtype=np.int64)
    jj = np.ascontiguousarray(jj, dtype=np.int64)
    d = np.empty(ii.shape, np.float64)
    s = np.empty(ii.shape, np.float64)
    st = lib().ora_gemm_sampled(_p(a.codes, ctypes.c_uint8), _p(a.scales_rm, ctypes.c_uint8), a.s_t,
                                _p(b.codes, ctypes.c_uint8), _p(b.scales_rm, ctypes.c_uint8), b.s_t, a.K,
                                _p(ii, ctypes.c_int64), _p(jj, ctypes.c_int64), ii.size, _p(d, ctypes.c_double),
                                _p(s, ctypes.c_double), nthreads or default_threads())
    if st != OK:
        raise ValueError(f"oracle gemm failed with status {st}")
    return d, s


def gelu_fwd(h_bits: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h_bits, dtype=np.uint16)
    g = np.empty_like(h)
    lib().ora_gelu_fwd(_p(h, ctypes.c_uint16), h.size, _p(g, ctypes.c_uint16))
    return g


def gelu_bwd(h_bits: np.ndarray, dg_bits: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h_bits, dtype=np.uint16)
    dg = np.ascontiguousarray(dg_bits, dtype=np.uint16)
    out = np.empty_like(h)
    lib().ora_gelu_bwd(_p(h, ctypes.c_uint16), _p(dg, ctypes.c_uint16), h.size, _p(out, ctypes.c_uint16))
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------------------------------
# MXFP4 (the pages' comparison format): blocks of 32, UE8M0 scales, no tensor scale
# ---------------------------------------------------------------------------------------
def ue8m0_of_amax(amax: float) -> int:
    """The UE8M0 code of a block with this amax: floor(log2 amax) - 2 + 127, in [0, 254]."""
    return int(lib().ora_ue8m0_of_amax(float(amax)))


def quantize_mx(x_bits: np.ndarray, mode: int = RNE, sr_seed: int = 0, stream_id: int = 0):
    """MXFP4 of a bf16 tensor [rows][cols] (uint16 bit patterns): codes [rows][cols/2] (even k in
    the low nibble) and UE8M0 scales [rows][cols/32]."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    rows, cols = x.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 32), np.uint8)
    st = lib().ora_quantize_mx(_p(x, ctypes.c_uint16), rows, cols, cols, mode, sr_seed, stream_id,
                               _p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8))
    if st != 0:
        raise ValueError(f"ora_quantize_mx: status {st}")
    return codes, scales


def dequantize_mx(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """MXFP4 form -> fp64 values [R][K]: E2M1(code) * 2^(scale - 127), exact."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    R, K = codes.shape[0], codes.shape[1] * 2
    out = np.empty((R, K), np.float64)
    lib().ora_dequantize_mx(_p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8), R, K, _p(out, ctypes.c_double))
    return out


def mx_scales_swizzled(scales: np.ndarray, K: int) -> np.ndarray:
    """Row-major MXFP4 scales [R][K/32] in the 128x4 tile layout of the block-scaled MMA."""
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    R = scales.shape[0]
    sw = np.empty(((R + 127) // 128) * 128 * ((K // 32 + 3) // 4) * 4, np.uint8)
    lib().ora_mx_scales_swizzle(_p(scales, ctypes.c_uint8), R, K, _p(sw, ctypes.c_uint8))
    return sw


def gemm_mx(a_codes, a_scales, b_codes, b_scales):
    """D = A * B^T in fp64 over dequantized MXFP4 operands (numpy's matmul as the dot-product
    step), plus sum_k |a_ik b_jk|."""
    A, B = dequantize_mx(a_codes, a_scales), dequantize_mx(b_codes, b_scales)
    return A @ B.T, np.abs(A) @ np.abs(B).T


# ---------------------------------------------------------------------------------------
# BF16 GEMM of the high-precision layers: the plain definition, in fp64
# ---------------------------------------------------------------------------------------
def gemm_bf16(a_bits: np.ndarray, b_bits: np.ndarray):
    """D = A * B^T in fp64 over bf16 operands given as uint16 bit patterns ([M][K], [N][K]);
    every bf16 value and every product is exact in fp64 (numpy's matmul as the dot-product step).
    Returns D and sum_k |a_ik b_jk|."""
    A = bf16_bits_to_f32(a_bits).astype(np.float64)
    B = bf16_bits_to_f32(b_bits).astype(np.float64)
    return A @ B.T, np.abs(A) @ np.abs(B).T
