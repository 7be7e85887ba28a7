"""Bit-exact parity of the CUDA quantizers against the CPU oracle: codes, swizzled scales
(padding included), 16x16 tile grids and the fp32 tensor scale, for every form the linear
layer uses (gist.science "Pretraining Large Language Models with NVFP4", 2.A and 2.B.2-4)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import assert_form_equal, nv, to_device_bf16

pytestmark = pytest.mark.gpu

SMALL = [(256, 256), (112, 528), (64, 1040), (1040, 48), (320, 256), (96, 160)]


def _x(rows, cols, seed, kind="act"):
    if kind == "act":
        t = synth.activations(rows, cols, seed=seed, outlier_frac=0.01)
    elif kind == "w":
        t = synth.weights(rows, cols, seed=seed)
    else:
        t = synth.grad_output(rows, cols, seed=seed)
    return t, synth.bf16_bits(t)


@pytest.mark.parametrize("rows,cols", SMALL + [(200, 320), (17, 64), (1, 16)])
@pytest.mark.parametrize("mode", [0, 1])
def test_row_form(rows, cols, mode):
    m = nv()
    t, bits = _x(rows, cols, seed=rows + cols)
    g = m.nvfp4_quantize(to_device_bf16(t), along=0, mode=mode, sr_seed=77, stream_id=1)
    q = oracle.quantize(bits, along=0, mode=mode, sr_seed=77, stream_id=1)
    assert_form_equal(g, q, f"row form {rows}x{cols} mode {mode}")


@pytest.mark.parametrize("rows,cols", SMALL)
@pytest.mark.parametrize("mode,rht", [(0, False), (0, True), (1, True), (1, False)])
def test_col_form(rows, cols, mode, rht):
    m = nv()
    t, bits = _x(rows, cols, seed=3, kind="grad" if mode else "act")
    g = m.nvfp4_quantize(to_device_bf16(t), along=1, mode=mode, rht=rht, rht_seed=5, sr_seed=9, stream_id=2)
    q = oracle.quantize(bits, along=1, mode=mode, rht=rht, rht_seed=5, sr_seed=9, stream_id=2)
    assert_form_equal(g, q, f"col form {rows}x{cols} mode {mode} rht {rht}")


@pytest.mark.parametrize("rows,cols", SMALL)
@pytest.mark.parametrize("along", [0, 1])
def test_16x16(rows, cols, along):
    m = nv()
    t, bits = _x(rows, cols, seed=1, kind="w")
    g = m.nvfp4_quantize(to_device_bf16(t), along=along, block=m.BLOCK_16x16)
    q = oracle.quantize(bits, along=along, block=oracle.BLOCK_16x16)
    assert_form_equal(g, q, f"16x16 along {along} {rows}x{cols}")


@pytest.mark.parametrize("rows,cols", SMALL)
@pytest.mark.parametrize("mode", [0, 1])
def test_dual_equals_two_single_calls(rows, cols, mode):
    m = nv()
    t, bits = _x(rows, cols, seed=11, kind="grad" if mode else "act")
    r, c = m.nvfp4_quantize_dual(to_device_bf16(t), mode=mode, rht_seed=13, sr_seed=21, stream_row=1, stream_col=2)
    qr = oracle.quantize(bits, along=0, mode=mode, sr_seed=21, stream_id=1)
    qc = oracle.quantize(bits, along=1, mode=mode, rht=True, rht_seed=13, sr_seed=21, stream_id=2)
    assert_form_equal(r, qr, "dual row")
    assert_form_equal(c, qc, "dual col")


@pytest.mark.parametrize("rows,cols", SMALL)
def test_weight_and_transpose(rows, cols):
    m = nv()
    t, bits = _x(rows, cols, seed=2, kind="w")
    wq, wqt = m.nvfp4_quantize_weight(to_device_bf16(t))
    q = oracle.quantize(bits, block=oracle.BLOCK_16x16)
    qt = oracle.transpose_2d(q)
    assert_form_equal(wq, q, "weight")
    assert_form_equal(wqt, qt, "weight transposed (fused)")
    wt2 = m.nvfp4_transpose_2d(wq)
    assert_form_equal(wt2, qt, "nvfp4_transpose_2d")


def test_empty_and_zero():
    m = nv()
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    g = m.nvfp4_quantize(x)
    torch.cuda.synchronize()
    assert g.tensor_scale.item() == 1.0
    z = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    g = m.nvfp4_quantize(z, along=1, rht=True)
    q = oracle.quantize(np.zeros((64, 64), np.uint16), along=1, rht=True)
    assert_form_equal(g, q, "zero tensor")


def test_nonfinite_is_flagged():
    m = nv()
    ws = m.Workspace()
    x = torch.ones((32, 32), dtype=torch.bfloat16, device="cuda")
    x[5, 7] = float("inf")
    m.nvfp4_quantize(x, ws=ws)
    assert m.nvfp4_poll(ws) == 7
    assert m.nvfp4_poll(ws) == 0          # flags clear after a poll
    x[5, 7] = float("nan")
    m.nvfp4_quantize_dual(x, ws=ws)
    assert m.nvfp4_poll(ws) == 7
    m.nvfp4_quantize(torch.ones((32, 32), dtype=torch.bfloat16, device="cuda"), ws=ws)
    assert m.nvfp4_poll(ws) == 0


@pytest.mark.parametrize("bits", [0x7F80, 0xFF80, 0x7FC0, 0xFFC1])   # +inf, -inf, NaN, negative NaN
@pytest.mark.parametrize("pos", [(0, 0), (5, 7), (31, 30), (16, 31)])  # both elements of a column pair
def test_nonfinite_is_flagged_by_the_rht_amax_pass(bits, pos):
    # the dual call's amax pass (plain amax as a NaN-propagating fp32 max, RHT amax alongside)
    m = nv()
    ws = m.Workspace()
    x = torch.ones((32, 32), dtype=torch.bfloat16, device="cuda")
    x.view(torch.int16)[pos] = bits - (1 << 16) if bits >= 1 << 15 else bits
    m.nvfp4_quantize_dual(x, ws=ws)
    assert m.nvfp4_poll(ws) == 7
    m.nvfp4_quantize_dual(torch.ones((32, 32), dtype=torch.bfloat16, device="cuda"), ws=ws)
    assert m.nvfp4_poll(ws) == 0


def test_leading_dimension():
    m = nv()
    t, bits = _x(64, 256, seed=4)
    big = torch.zeros((64, 384), dtype=torch.bfloat16)
    big[:, :256] = t
    g = m.nvfp4_quantize(to_device_bf16(big)[:, :256], along=0)
    q = oracle.quantize(bits, along=0)
    assert_form_equal(g, q, "ld > cols")


# ---- the full-size operands of the 8192 x 5120 x 20480 layer ---------------------------------
def test_full_size_activation_dual():
    m = nv()
    t = synth.activations(synth.TOKENS, synth.D_IN, seed=0, outlier_frac=0.001)
    bits = synth.bf16_bits(t)
    r, c = m.nvfp4_quantize_dual(to_device_bf16(t), mode=0, rht_seed=0)
    assert_form_equal(r, oracle.quantize(bits, along=0), "X row form")
    assert_form_equal(c, oracle.quantize(bits, along=1, rht=True, rht_seed=0), "X^T RHT form")


def test_full_size_weight():
    m = nv()
    t = synth.weights(synth.D_OUT, synth.D_IN, seed=1)
    bits = synth.bf16_bits(t)
    wq, wqt = m.nvfp4_quantize_weight(to_device_bf16(t))
    q = oracle.quantize(bits, block=oracle.BLOCK_16x16)
    assert_form_equal(wq, q, "W 16x16")
    assert_form_equal(wqt, oracle.transpose_2d(q), "W^T")


def test_full_size_grad_dual_sr():
    m = nv()
    t = synth.grad_output(synth.TOKENS, synth.D_OUT, seed=2)
    bits = synth.bf16_bits(t)
    r, c = m.nvfp4_quantize_dual(to_device_bf16(t), mode=1, rht_seed=0, sr_seed=0, stream_row=1, stream_col=2)
    assert_form_equal(r, oracle.quantize(bits, along=0, mode=1, sr_seed=0, stream_id=1), "dY row form (SR)")
    assert_form_equal(c, oracle.quantize(bits, along=1, mode=1, rht=True, rht_seed=0, sr_seed=0, stream_id=2),
                      "dY^T RHT form (SR)")
