"""The BF16 path of the layers the recipe keeps in high precision (gist.science "Pretraining Large
Language Models with NVFP4", 2.B.1): the tcgen05 kind::f16 GEMM, the bf16 transpose and the BF16
linear layer against the oracle's fp64 product of the same bf16 values.

Tolerance (from the arithmetic): bf16 x bf16 products are exact in fp32, and the fp32
accumulation of K of them errs by at most gamma_K * sum_k |a_k b_k| with gamma_K = K u / (1 - K u);
u = 2^-23 (one fp32 ulp, allowing truncating adds in the tensor core), plus 2^-8 |D_ref| for a
bf16 output's final rounding.  Small-integer operands are exact and compared bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import bf16_to_f64, nv, to_device_bf16

pytestmark = pytest.mark.gpu


def _check(got, ref, sabs, K, bf16_out, what):
    u = 2.0 ** -23
    gamma = K * u / (1 - K * u)
    tol = gamma * sabs + (2.0 ** -8 * np.abs(ref) if bf16_out else 0.0) + 1e-30
    err = np.abs(got.astype(np.float64) - ref)
    bad = err > tol
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} outside; worst ratio {float(np.max(err / tol)):.3g}"


@pytest.mark.parametrize("M,N,K", [(256, 256, 256), (512, 768, 1280), (100, 200, 64), (1, 8, 8), (300, 520, 136),
                                   (128, 256, 2048)])
@pytest.mark.parametrize("out", ["bf16", "fp32"])
def test_bf16_gemm_within_accumulation_bound(M, N, K, out):
    m = nv()
    a = synth.activations(M, K, seed=M + K, outlier_frac=0.01)
    b = synth.weights(N, K, seed=N + K)
    dt = torch.bfloat16 if out == "bf16" else torch.float32
    d = m.nvfp4_bf16_gemm(to_device_bf16(a), to_device_bf16(b), out_dtype=dt)
    ref, sabs = oracle.gemm_bf16(synth.bf16_bits(a), synth.bf16_bits(b))
    got = bf16_to_f64(d) if out == "bf16" else d.cpu().numpy()
    _check(got, ref, sabs, K, out == "bf16", f"bf16 GEMM {M}x{N}x{K} {out}")


@pytest.mark.parametrize("M,N,K", [(256, 512, 64), (384, 256, 128), (130, 136, 32)])
def test_bf16_gemm_exact_on_small_integers(M, N, K):
    # |a|, |b| <= 8 and K <= 128: every partial sum is an integer below 2^24, exact in fp32
    m = nv()
    g = torch.Generator().manual_seed(M + N + K)
    a = torch.randint(-8, 9, (M, K), generator=g).to(torch.bfloat16)
    b = torch.randint(-8, 9, (N, K), generator=g).to(torch.bfloat16)
    d = m.nvfp4_bf16_gemm(to_device_bf16(a), to_device_bf16(b), out_dtype=torch.float32)
    ref, _ = oracle.gemm_bf16(synth.bf16_bits(a), synth.bf16_bits(b))
    assert np.array_equal(d.cpu().numpy().astype(np.float64), ref)


@pytest.mark.parametrize("rows,cols", [(64, 64), (200, 136), (8, 520), (1024, 24)])
def test_bf16_transpose_exact(rows, cols):
    m = nv()
    x = synth.activations(rows, cols, seed=rows)
    xt = m.nvfp4_bf16_transpose(to_device_bf16(x))
    assert torch.equal(xt.cpu(), x.t().contiguous())


@pytest.mark.parametrize("T,d,n", [(256, 320, 512), (192, 128, 264)])
def test_bf16_linear_layer(T, d, n):
    m = nv()
    x = synth.activations(T, d, seed=0, outlier_frac=0.01)
    w = synth.weights(n, d, seed=1)
    dy = synth.grad_output(T, n, seed=2)
    lay = m.LinearBF16(T, d, n)
    xd, wd, dyd = map(to_device_bf16, (x, w, dy))
    y = lay.fwd(xd, wd)
    dx, dw = lay.bwd(xd, wd, dyd)
    assert m.nvfp4_poll(lay.ws) == 0
    xb, wb, dyb = map(synth.bf16_bits, (x, w, dy))
    ref, s = oracle.gemm_bf16(xb, wb)
    _check(bf16_to_f64(y), ref, s, d, True, "Y = X W^T")
    ref, s = oracle.gemm_bf16(dyb, np.ascontiguousarray(wb.T))
    _check(bf16_to_f64(dx), ref, s, n, True, "dX = dY W")
    ref, s = oracle.gemm_bf16(np.ascontiguousarray(dyb.T), np.ascontiguousarray(xb.T))
    _check(dw.cpu().numpy(), ref, s, T, False, "dW = dY^T X")
