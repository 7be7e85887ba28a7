"""nvfp4_quantize_noalloc: the quantize entry point for callers that cannot allocate device
memory (their host owns all of it and offers no allocation hook, so they cannot pass a
workspace).  Called through the C ABI, its output must equal that of nvfp4_quantize with a
caller-provided workspace, bit for bit -- the same tolerance as every quantize parity test --
on two calls in a row, so leftovers in the shared scratch array cannot change a result."""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _entry():
    import nvfp4_bit_quantized_02_b200 as nv
    f = nv.lib().nvfp4_quantize_noalloc
    c = ctypes
    f.argtypes = [c.c_void_p, c.c_int64, c.c_int64, c.c_int64, c.c_int, c.c_int, c.c_int, c.c_int, c.c_uint64,
                  c.c_uint64, c.c_uint32, c.POINTER(nv.CTensor), c.c_void_p]
    f.restype = c.c_int
    return nv, f


def _same(nv, a, b):
    torch.cuda.synchronize()
    n = a.rows * (a.k // 2)
    assert torch.equal(a.codes[:n], b.codes[:n])
    s = nv.lib().nvfp4_scales_bytes(a.rows, a.k)
    assert torch.equal(a.scales[:s], b.scales[:s])
    assert a.tensor_scale.view(torch.int32).item() == b.tensor_scale.view(torch.int32).item()


CASES = [
    # (source, along, mode, block, rht)
    ("act", 0, 0, 0, False),
    ("grad", 1, 1, 0, True),
    ("weight", 0, 0, 1, False),
]


@pytest.mark.parametrize("kind,along,mode,block,rht", CASES)
def test_noalloc_matches_workspace_entry_point(kind, along, mode, block, rht):
    nv, f = _entry()
    rows, cols = 192, 320
    src = {"act": lambda s: synth.activations(rows, cols, seed=s, outlier_frac=0.01),
           "grad": lambda s: synth.grad_output(rows, cols, seed=s),
           "weight": lambda s: synth.weights(rows, cols, seed=s)}[kind]
    R, K = (cols, rows) if along else (rows, cols)
    for call, seed in enumerate((5, 6)):     # two calls in a row, different inputs
        x = src(seed).cuda()
        ref = nv.nvfp4_quantize(x, along=along, mode=mode, block=block, rht=rht, rht_seed=3, sr_seed=9, stream_id=2)
        out = nv.NVFP4Tensor.empty(R, K, block)
        ct = out.c()
        st = f(ctypes.c_void_p(x.data_ptr()), rows, cols, cols, along, mode, block, int(rht), 3, 9, 2, ctypes.byref(ct),
               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0, f"call {call}: status {st}"
        _same(nv, out, ref)


def _call(nv, f, x, rows, cols, along, mode, block, rht, out):
    ct = out.c()
    xp = ctypes.c_void_p(x.data_ptr()) if x is not None and x.numel() else None
    st = f(xp, rows, cols, cols, along, mode, block, int(rht), 3, 9, 2, ctypes.byref(ct),
           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


def _poll(nv):
    p = nv.lib().nvfp4_poll_noalloc
    p.argtypes = [ctypes.c_void_p]
    p.restype = ctypes.c_int
    return p(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_empty_and_refused_shapes_match_workspace_entry_point():
    # zero rows: status 0 and a tensor scale of 1, as nvfp4_quantize gives; a shape that
    # nvfp4_quantize refuses before any device work is refused with the same status
    nv, f = _entry()
    out = nv.NVFP4Tensor.empty(16, 64, 0)
    out.tensor_scale.fill_(7.0)
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    assert _call(nv, f, x, 0, 64, 0, 0, 0, False, out) == 0
    torch.cuda.synchronize()
    assert out.tensor_scale.item() == 1.0
    ws = nv.Workspace()
    x = torch.ones((24, 64), dtype=torch.bfloat16, device="cuda")    # along = 1 needs rows % 16 == 0
    ref_st = nv.lib().nvfp4_quantize(ctypes.c_void_p(x.data_ptr()), 24, 64, 64, 1, 0, 0, 0, 3, 9, 2,
                                     ctypes.byref(nv.NVFP4Tensor.empty(64, 24, 0).c()), ws.ptr, None)
    assert ref_st == 3
    assert _call(nv, f, x, 24, 64, 1, 0, 0, False, nv.NVFP4Tensor.empty(64, 24, 0)) == ref_st


def test_noalloc_poll_reports_and_clears_device_flags():
    # a non-finite input is flagged in the library's array and reported once by the poll
    nv, f = _entry()
    assert _poll(nv) == 0
    x = torch.ones((32, 32), dtype=torch.bfloat16, device="cuda")
    x[3, 5] = float("nan")
    assert _call(nv, f, x, 32, 32, 0, 0, 0, False, nv.NVFP4Tensor.empty(32, 32, 0)) == 0
    assert _poll(nv) == 7
    assert _poll(nv) == 0
    x[3, 5] = 1.0
    assert _call(nv, f, x, 32, 32, 0, 0, 0, False, nv.NVFP4Tensor.empty(32, 32, 0)) == 0
    assert _poll(nv) == 0
