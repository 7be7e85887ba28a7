"""The one-FFN training step (up-projection, GeLU, down-projection; forward and backward) on the
GPU against the oracle, and the GeLU kernels on their own.

Forward:  H = X W1^T,  G = GeLU(H),  Y = G W2^T.
Backward: dG = dY W2,  dW2 = dY^T G,  dH = dG * GeLU'(H),  dX = dH W1,  dW1 = dH^T X.
Every GEMM is an NVFP4 linear of the pages' recipe (gist.science "Pretraining Large Language
Models with NVFP4", 2.B: 16x16 weights reused transposed, RHT on the wgrad operands, SR on the
gradients); the GeLU is the glue between them (not in the pages; exact erf form).

Quantization decisions depend on the exact input bits, so the chain is checked link by link:
each GPU stage is compared with the oracle fed that stage's GPU inputs.  Quantized forms must
match bit for bit, GEMM outputs stay within |D - D_ref| <= 1e-5 sum|a b| (+ 2^-8 |D_ref| for
bf16), GeLU outputs within one bf16 step."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import assert_form_equal, bf16_to_f64, check_gemm, check_gemm_sampled, nv, to_device_bf16

pytestmark = pytest.mark.gpu


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _ulps(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    def line(x):
        x = x.astype(np.int32)
        return np.where(x & 0x8000, -(x & 0x7FFF), x & 0x7FFF)
    return np.abs(line(a) - line(b))


def _gelu_inputs(n: int, seed: int) -> torch.Tensor:
    g = torch.Generator(device="cpu").manual_seed(seed)
    parts = [torch.randn(n // 4, generator=g) * s for s in (1e-3, 0.5, 2.0, 6.0)]
    special = torch.tensor([0.0, -0.0, 1.0, -1.0, -4.0, -6.0, -9.0, -12.0, -20.0, 10.0, 40.0, 1e-30, -1e-30])
    x = torch.cat(parts + [special])[:n] if n >= special.numel() else special[:n]
    if x.numel() < n:
        x = torch.cat([x, torch.randn(n - x.numel(), generator=g)])
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("n", [1, 7, 8, 1000, 65536 + 13])
def test_gelu_kernels_within_one_bf16_step(n):
    m = nv()
    h = _gelu_inputs(n, seed=n)
    dg = (torch.randn(n, generator=torch.Generator().manual_seed(n + 1)) * 1e-3).to(torch.bfloat16)
    g = m.nvfp4_gelu_fwd(to_device_bf16(h))
    dh = m.nvfp4_gelu_bwd(to_device_bf16(h), to_device_bf16(dg))
    hb, dgb = synth.bf16_bits(h), synth.bf16_bits(dg)
    for what, got, ref in (("fwd", _bits(g), oracle.gelu_fwd(hb)), ("bwd", _bits(dh), oracle.gelu_bwd(hb, dgb))):
        d = _ulps(got, ref)
        assert d.max() <= 1, f"{what}: {int((d > 1).sum())} elements more than one bf16 step off, worst {int(d.max())}"
        if n >= 1000:
            assert np.mean(d == 0) > 0.98, what


def test_gelu_kernels_on_every_finite_bf16_input():
    # every finite bf16 h (65280 values), forward and backward at three gradient scales: within
    # one bf16 step of the exactly rounded fp64 values, and nearly all exact
    m = nv()
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = (bits.astype(np.uint32) << 16).view(np.float32)
    bits = bits[np.isfinite(vals)]
    h = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
    got = _bits(m.nvfp4_gelu_fwd(to_device_bf16(h)))
    d = _ulps(got, oracle.gelu_fwd(bits))
    assert d.max() <= 1 and np.mean(d == 0) > 0.999, (int(d.max()), float(np.mean(d == 0)))
    for scale in (1e-3, 1.0, 3e4):
        dg = torch.full_like(h, scale)
        got = _bits(m.nvfp4_gelu_bwd(to_device_bf16(h), to_device_bf16(dg)))
        d = _ulps(got, oracle.gelu_bwd(bits, synth.bf16_bits(dg)))
        assert d.max() <= 1 and np.mean(d == 0) > 0.999, (scale, int(d.max()), float(np.mean(d == 0)))


@pytest.mark.parametrize("rows,cols", [(64, 256), (160, 512)])
def test_gelu_amax_kernels(rows, cols):
    # the fused kernels' outputs stay within one bf16 step of the oracle, and the amax words they
    # leave in the workspace are exactly the oracle's amax of those outputs (plain and after the
    # RHT along rows)
    m = nv()
    g_ = torch.Generator().manual_seed(rows + cols)
    h = (torch.randn(rows, cols, generator=g_) * 2.0).to(torch.bfloat16)
    dg = (torch.randn(rows, cols, generator=g_) * 1e-3).to(torch.bfloat16)
    hb = synth.bf16_bits(h)
    for bwd in (False, True):
        ws = m.Workspace()
        if bwd:
            out = m.nvfp4_gelu_bwd_amax(to_device_bf16(h), to_device_bf16(dg), rht_seed=7, ws=ws)
            ref = oracle.gelu_bwd(hb, synth.bf16_bits(dg))
        else:
            out = m.nvfp4_gelu_fwd_amax(to_device_bf16(h), rht_seed=7, ws=ws)
            ref = oracle.gelu_fwd(hb)
        ob = _bits(out).reshape(rows, cols)
        assert _ulps(ob.reshape(-1), np.asarray(ref).reshape(-1)).max() <= 1
        words = ws.amax_words().cpu().numpy().view(np.float32)
        assert words[0] == np.float32(oracle.quantize(ob).amax), "plain amax"
        assert words[1] == np.float32(oracle.quantize(ob, along=1, rht=True, rht_seed=7).amax), "RHT amax"


def _check_linear_forms(ctx, xb, wb, rht_seed):
    xq = oracle.quantize(xb)
    xq_rht = oracle.quantize(xb, along=1, rht=True, rht_seed=rht_seed)
    wq = oracle.quantize(wb, block=oracle.BLOCK_16x16)
    wqt = oracle.transpose_2d(wq)
    for name, q in (("xq", xq), ("xq_rht", xq_rht), ("wq", wq), ("wqt", wqt)):
        assert_form_equal(getattr(ctx, name), q, name)
    return dict(xq=xq, xq_rht=xq_rht, wq=wq, wqt=wqt)


def _check_grad_forms(ctx, dyb, rht_seed, sr_seed):
    dyq = oracle.quantize(dyb, mode=oracle.SR, sr_seed=sr_seed, stream_id=1)
    dyq_rht = oracle.quantize(dyb, along=1, mode=oracle.SR, rht=True, rht_seed=rht_seed, sr_seed=sr_seed, stream_id=2)
    assert_form_equal(ctx.dyq, dyq, "dyq")
    assert_form_equal(ctx.dyq_rht, dyq_rht, "dyq_rht")
    return dyq, dyq_rht


def _chain(T, d, f, fused, full_check: bool):
    """The FFN step on the GPU, every link checked against the oracle fed that link's GPU inputs:
    whole quantized forms bit for bit; GEMM outputs in full (full_check) or on the sampled
    positions of the full-size checks."""
    m = nv()
    rht_seed = 0
    x = synth.activations(T, d, seed=0, outlier_frac=0.01 if full_check else 0.001)
    w1 = synth.weights(f, d, seed=1)
    w2 = synth.weights(d, f, seed=3)
    dy = synth.grad_output(T, d, seed=4)
    up = m.LinearContext(T, d, f, rht_seed=rht_seed)
    down = m.LinearContext(T, f, d, rht_seed=rht_seed)
    seeds = iter(range(1, 100))

    def gemm_check(out, a, b, bf, what):
        if full_check:
            ref, s = oracle.gemm_full(a, b)
            check_gemm(bf16_to_f64(out) if bf else out.cpu().numpy(), ref, s, bf, what)
        else:
            check_gemm_sampled(out, a, b, bf, what, seed=next(seeds))

    # forward
    h = m.nvfp4_linear_fwd(up, to_device_bf16(x), to_device_bf16(w1))
    o_up = _check_linear_forms(up, synth.bf16_bits(x), synth.bf16_bits(w1), rht_seed)
    gemm_check(h, o_up["xq"], o_up["wq"], True, "H = X W1^T")

    if fused:   # the GeLU reduces G's amax; the down-projection skips its amax pass
        g = m.nvfp4_gelu_fwd_amax(h, rht_seed=rht_seed, ws=down.ws)
        down.amax_ready = True
    else:
        g = m.nvfp4_gelu_fwd(h)
    hb = _bits(h)
    assert _ulps(_bits(g), oracle.gelu_fwd(hb)).max() <= 1, "G = GeLU(H)"

    y = m.nvfp4_linear_fwd(down, g, to_device_bf16(w2))
    gb = _bits(g)
    o_down = _check_linear_forms(down, gb, synth.bf16_bits(w2), rht_seed)
    gemm_check(y, o_down["xq"], o_down["wq"], True, "Y = G W2^T")
    del gb

    # backward through the down-projection
    dg, dw2 = m.nvfp4_linear_bwd(down, to_device_bf16(dy), 5)
    dyq, dyq_rht = _check_grad_forms(down, synth.bf16_bits(dy), rht_seed, 5)
    gemm_check(dg, dyq, o_down["wqt"], True, "dG = dY W2")
    gemm_check(dw2, dyq_rht, o_down["xq_rht"], False, "dW2 = dY^T G")
    del o_down, dyq, dyq_rht, dw2

    if fused:
        dh = m.nvfp4_gelu_bwd_amax(h, dg, rht_seed=rht_seed, ws=up.ws)
        up.amax_ready = True
    else:
        dh = m.nvfp4_gelu_bwd(h, dg)
    assert _ulps(_bits(dh), oracle.gelu_bwd(hb, _bits(dg))).max() <= 1, "dH = dG GeLU'(H)"
    del hb

    # backward through the up-projection
    dx, dw1 = m.nvfp4_linear_bwd(up, dh, 6)
    dhq, dhq_rht = _check_grad_forms(up, _bits(dh), rht_seed, 6)
    gemm_check(dx, dhq, o_up["wqt"], True, "dX = dH W1")
    gemm_check(dw1, dhq_rht, o_up["xq_rht"], False, "dW1 = dH^T X")
    assert m.nvfp4_poll(up.ws) == 0 and m.nvfp4_poll(down.ws) == 0
    assert not up.amax_ready and not down.amax_ready


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("T,d,f", [(256, 128, 512), (128, 192, 256)])
def test_ffn_step_chain(T, d, f, fused):
    _chain(T, d, f, fused, full_check=True)


@pytest.mark.parametrize("fused", [False, True])
def test_ffn_step_chain_full_size(fused):
    # the one-FFN training step at its benchmark size: T = 16384 tokens, 5120 -> 20480 -> 5120
    # (the wgrad forms have K = 16384); X with 0.1 % outlier channels
    _chain(16384, 5120, 20480, fused, full_check=False)
