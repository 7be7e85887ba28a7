"""The C-ABI library loads on a machine without a GPU and exports every entry point that
include/nvfp4.h declares; host-only calls (sizes, status strings) and argument validation
work without touching a device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    import nvfp4_bit_quantized_02_b200 as nv
    if not os.path.exists(nv.LIB_PATH):
        from nvfp4_bit_quantized_02_b200.csrc import build as b
        b.build()
    return nv.lib()


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 15
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing


def test_sizes(L):
    assert L.nvfp4_codes_bytes(8192, 5120) == 8192 * 2560
    assert L.nvfp4_scales_bytes(8192, 5120) == 8192 * 320
    assert L.nvfp4_scales_bytes(200, 48) == 256 * 4       # rows to 128, K/16 to a multiple of 4
    assert L.nvfp4_tile_scales_bytes(20480, 5120) == 1280 * 320
    assert L.nvfp4_workspace_bytes() == 256
    assert L.nvfp4_codes_bytes(0, 64) == 0


def test_status_strings(L):
    for s in range(11):
        assert L.nvfp4_status_string(s)
    assert L.nvfp4_status_string(0) == b"ok"
    assert L.nvfp4_version() >= 1


def test_validation_before_any_device_work(L):
    import nvfp4_bit_quantized_02_b200 as nv
    t = nv.CTensor(16, 16, 0, 16, 0, 0, 0, 0)
    ws = ctypes.c_void_p(16)
    x = ctypes.c_void_p(16)
    # cols not a multiple of 16
    assert L.nvfp4_quantize(x, 32, 24, 24, 0, 0, 0, 0, 0, 0, 0, ctypes.byref(t), ws, None) == 3
    # misaligned input
    assert L.nvfp4_quantize(ctypes.c_void_p(18), 32, 32, 32, 0, 0, 0, 0, 0, 0, 0, ctypes.byref(t), ws, None) == 2
    # bad enums / RHT on a non-wgrad form
    assert L.nvfp4_quantize(x, 32, 32, 32, 2, 0, 0, 0, 0, 0, 0, ctypes.byref(t), ws, None) == 4
    assert L.nvfp4_quantize(x, 32, 32, 32, 0, 0, 0, 1, 0, 0, 0, ctypes.byref(t), ws, None) == 4
    # 16x16 without tile scales
    assert L.nvfp4_quantize(x, 32, 32, 32, 0, 0, 1, 0, 0, 0, 0, ctypes.byref(t), ws, None) == 1
    # missing workspace
    assert L.nvfp4_quantize(x, 32, 32, 32, 0, 0, 0, 0, 0, 0, 0, ctypes.byref(t), None, None) == 5
    # along=1 needs rows % 16
    assert L.nvfp4_quantize(x, 24, 32, 32, 1, 0, 0, 0, 0, 0, 0, ctypes.byref(t), ws, None) == 3
    # GEMM: K mismatch, K % 32, null output, misaligned ldd
    a = nv.CTensor(16, 16, 0, 16, 128, 64, 0, 0)
    b = nv.CTensor(16, 16, 0, 16, 128, 96, 0, 0)
    d = ctypes.c_void_p(16)
    assert L.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), d, 128, 0, ws, None) == 4
    b.k = 48
    a.k = 48
    assert L.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), d, 128, 0, ws, None) == 3
    a.k = b.k = 64
    assert L.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), None, 128, 0, ws, None) == 1
    assert L.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), d, 129, 0, ws, None) == 2
    assert L.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), d, 100, 0, ws, None) == 3
    # the amax epilogue: its workspace, M % 16, bf16 row alignment
    assert L.nvfp4_gemm_amax(ctypes.byref(a), ctypes.byref(b), d, 128, 0, None, ws, None) == 5
    a.rows = 120
    assert L.nvfp4_gemm_amax(ctypes.byref(a), ctypes.byref(b), d, 128, 0, ws, ws, None) == 3
    a.rows = 128
    assert L.nvfp4_gemm_amax(ctypes.byref(a), ctypes.byref(b), d, 132, 0, ws, ws, None) == 2
    # sizes past the fixed limit (2^30 rows or K) are refused before any device work
    a.rows = (1 << 30) + 16
    assert L.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), d, 128, 0, ws, None) == 10
    assert L.nvfp4_gemm_amax(ctypes.byref(a), ctypes.byref(b), d, 128, 0, ws, ws, None) == 10
    a.rows = 128
    # linear: shapes must be multiples of 64
    ctx = nv.CLinearCtx()
    ctx.T, ctx.d, ctx.n, ctx.ws = 100, 64, 64, 16
    assert L.nvfp4_linear_fwd(x, x, x, ctypes.byref(ctx), None) == 3


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import nvfp4_bit_quantized_02_b200 as nv
    monkeypatch.setattr(nv, "_L", None)
    monkeypatch.setattr(nv, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        nv.lib()


def test_shard_entry_points_validate(L):
    import nvfp4_bit_quantized_02_b200 as nv
    t = nv.CTensor(16, 16, 0, 16, 0, 0, 0, 0)
    x, ws = ctypes.c_void_p(16), ctypes.c_void_p(16)
    assert L.nvfp4_workspace_amax_offset() == 4
    # amax: no workspace; rows not a multiple of 16 with the RHT
    assert L.nvfp4_amax(x, 32, 32, 32, 1, 0, None, None) == 5
    assert L.nvfp4_amax(x, 24, 32, 32, 1, 0, ws, None) == 3
    # shard: offset not a multiple of 16; shard past the end of the tensor; negative offset
    assert L.nvfp4_quantize_dual_shard(x, 32, 32, 32, 8, 64, 0, 0, 0, 1, 2, ctypes.byref(t), ctypes.byref(t), ws, None) == 3
    assert L.nvfp4_quantize_dual_shard(x, 32, 32, 32, 48, 64, 0, 0, 0, 1, 2, ctypes.byref(t), ctypes.byref(t), ws, None) == 3
    assert L.nvfp4_quantize_dual_shard(x, 32, 32, 32, -16, 64, 0, 0, 0, 1, 2, ctypes.byref(t), ctypes.byref(t), ws, None) == 3


def test_gelu_amax_entry_points_validate(L):
    h, ws = ctypes.c_void_p(16), ctypes.c_void_p(16)
    assert L.nvfp4_gelu_fwd_amax(h, h, 32, 32, 0, None, None) == 5       # no workspace
    assert L.nvfp4_gelu_fwd_amax(h, h, 24, 32, 0, ws, None) == 3         # rows % 16
    assert L.nvfp4_gelu_bwd_amax(h, None, h, 32, 32, 0, ws, None) == 1    # no dg
    assert L.nvfp4_gelu_bwd_amax(h, h, ctypes.c_void_p(18), 32, 32, 0, ws, None) == 2   # misaligned output


def test_gemm_size_limits_and_degenerate_shapes(L):
    # sizes past the GEMM's 2^30 limit per dimension are refused before any device work; so are
    # empty GEMMs (M or N of 0, K of 0)
    import nvfp4_bit_quantized_02_b200 as nv
    ws, d = ctypes.c_void_p(16), ctypes.c_void_p(16)
    big = (1 << 30) + 64
    for (M, N, K, want) in [(big, 128, 64, 10), (128, big, 64, 10), (128, 128, big - 32, 10),
                            (0, 128, 64, 3), (128, 0, 64, 3), (128, 128, 0, 3)]:
        a = nv.CTensor(16, 16, 0, 16, M, K, 0, 0)
        b = nv.CTensor(16, 16, 0, 16, N, K, 0, 0)
        assert L.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), d, max(N, 8), 0, ws, None) == want, (M, N, K)
