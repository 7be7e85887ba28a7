"""The whole NVFP4 linear layer (quantize + fprop, dgrad, wgrad GEMMs) on the GPU against the
oracle composed from the pages' steps (gist.science "Pretraining Large Language Models with
NVFP4", 2.B: 16x16 weights reused transposed, RHT on the wgrad inputs, SR on gradients).

Small shapes are checked in full; the 8192 x 5120 x 20480 layer of the benchmark is checked
on every element of 8 full 128x128 output tiles (four corners, the centre and three seeded
random tiles) plus 65536 seeded random elements of each GEMM output."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import assert_form_equal, bf16_to_f64, check_gemm, check_gemm_sampled, nv, to_device_bf16

pytestmark = pytest.mark.gpu


def _oracle_layer(xb, wb, dyb, rht_seed, sr_seed):
    xq = oracle.quantize(xb)
    xq_rht = oracle.quantize(xb, along=1, rht=True, rht_seed=rht_seed)
    wq = oracle.quantize(wb, block=oracle.BLOCK_16x16)
    wqt = oracle.transpose_2d(wq)
    dyq = oracle.quantize(dyb, mode=oracle.SR, sr_seed=sr_seed, stream_id=1)
    dyq_rht = oracle.quantize(dyb, along=1, mode=oracle.SR, rht=True, rht_seed=rht_seed, sr_seed=sr_seed, stream_id=2)
    return dict(xq=xq, xq_rht=xq_rht, wq=wq, wqt=wqt, dyq=dyq, dyq_rht=dyq_rht)


def _run_gpu(T, d, n, x, w, dy, rht_seed, sr_seed):
    m = nv()
    ctx = m.LinearContext(T, d, n, rht_seed=rht_seed)
    y = m.nvfp4_linear_fwd(ctx, to_device_bf16(x), to_device_bf16(w))
    dx, dw = m.nvfp4_linear_bwd(ctx, to_device_bf16(dy), sr_seed)
    assert m.nvfp4_poll(ctx.ws) == 0
    return ctx, y, dx, dw


@pytest.mark.parametrize("T,d,n", [(256, 256, 512), (192, 320, 128)])
def test_small_layer_full_check(T, d, n):
    x = synth.activations(T, d, seed=0, outlier_frac=0.01)
    w = synth.weights(n, d, seed=1)
    dy = synth.grad_output(T, n, seed=2)
    xb, wb, dyb = map(synth.bf16_bits, (x, w, dy))
    ctx, y, dx, dw = _run_gpu(T, d, n, x, w, dy, rht_seed=3, sr_seed=4)
    o = _oracle_layer(xb, wb, dyb, 3, 4)
    for name in o:
        assert_form_equal(getattr(ctx, name), o[name], name)
    ref, s = oracle.gemm_full(o["xq"], o["wq"])
    check_gemm(bf16_to_f64(y), ref, s, True, "fprop")
    ref, s = oracle.gemm_full(o["dyq"], o["wqt"])
    check_gemm(bf16_to_f64(dx), ref, s, True, "dgrad")
    ref, s = oracle.gemm_full(o["dyq_rht"], o["xq_rht"])
    check_gemm(dw.cpu().numpy(), ref, s, False, "wgrad")


def test_full_size_layer_sampled():
    T, d, n = synth.TOKENS, synth.D_IN, synth.D_OUT
    x = synth.activations(T, d, seed=0, outlier_frac=0.001)
    w = synth.weights(n, d, seed=1)
    dy = synth.grad_output(T, n, seed=2)
    ctx, y, dx, dw = _run_gpu(T, d, n, x, w, dy, rht_seed=0, sr_seed=0)
    o = _oracle_layer(*map(synth.bf16_bits, (x, w, dy)), 0, 0)
    for name in o:
        assert_form_equal(getattr(ctx, name), o[name], name)
    for what, out, a, b, bf in (("fprop", y, "xq", "wq", True), ("dgrad", dx, "dyq", "wqt", True),
                                ("wgrad", dw, "dyq_rht", "xq_rht", False)):
        check_gemm_sampled(out, o[a], o[b], bf, what, seed={"fprop": 1, "dgrad": 2, "wgrad": 3}[what])


def test_cached_weight_path_identical():
    m = nv()
    T, d, n = 128, 256, 256
    x, w = synth.activations(T, d, seed=5), synth.weights(n, d, seed=6)
    ctx = m.LinearContext(T, d, n)
    y1 = m.nvfp4_linear_fwd(ctx, to_device_bf16(x), to_device_bf16(w)).clone()
    ctx.w_cached = True
    y2 = m.nvfp4_linear_fwd(ctx, to_device_bf16(x), None)
    assert torch.equal(y1, y2)
