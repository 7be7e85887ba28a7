"""The tcgen05 block-scaled FP4 GEMM against the oracle's fp64 GEMM over the same quantized
operands (taken from the oracle and uploaded).  Exact cases use power-of-two scales so every
product and partial sum is representable: they pin the nibble order, the scale-tile layout and
the TMEM scale placement bit for bit.  Random cases use the tolerance
|D - D_ref| <= 1e-5 * sum_k |a_k b_k| (+ 2^-8 |D_ref| for bf16 output)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import bf16_to_f64, check_gemm, make_form, nv, upload_form

pytestmark = pytest.mark.gpu

POW2_SCALES = np.array([0x30, 0x38, 0x40], np.uint8)    # 0.5, 1, 2


def _exact_operand(rng, R, K):
    nib = rng.integers(0, 16, size=(R, K), dtype=np.uint8)
    sc = rng.choice(POW2_SCALES, size=(R, K // 16))
    return make_form(R, K, nib, sc, 0.125)


@pytest.fixture(params=["1sm", "2sm"])
def variant(request, monkeypatch):
    # the library reads NVFP4_GEMM_VARIANT on every call: 1sm forces the 1-SM kernel; otherwise
    # the SM-pair kernel runs for M >= 256 and the 1-SM kernel below that
    monkeypatch.setenv("NVFP4_GEMM_VARIANT", request.param)
    return request.param


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (128, 256, 256), (256, 512, 1024), (384, 256, 512),
                                   (200, 328, 96), (1, 8, 32), (130, 136, 160), (512, 384, 2048), (300, 200, 96)])
def test_exact_dyadic(M, N, K, variant):
    m = nv()
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    a, b = _exact_operand(rng, M, K), _exact_operand(rng, N, K)
    d = m.nvfp4_gemm(upload_form(a), upload_form(b), out_dtype=torch.float32)
    ref, _ = oracle.gemm_full(a, b)
    got = d.cpu().numpy().astype(np.float64)
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} differ; first {bad[0].tolist()}: gpu {got[tuple(bad[0])]} ref {ref[tuple(bad[0])]}"


def test_one_hot_probes_pin_layout(variant):
    # A row m has a single nonzero element at k = (37 m) % K with a distinct scale per row;
    # D[m][:] is then that element times column k of B: any error in the nibble order or in
    # the position of a scale shows up as a wrong row
    m = nv()
    M, N, K = 256, 256, 512
    rng = np.random.default_rng(0)
    nib = np.zeros((M, K), np.uint8)
    ks = (37 * np.arange(M)) % K
    nib[np.arange(M), ks] = rng.integers(1, 8, M)
    sc = np.full((M, K // 16), 0x38, np.uint8)
    sc[np.arange(M), ks // 16] = rng.choice(POW2_SCALES, M)
    a = make_form(M, K, nib, sc, 1.0)
    b = _exact_operand(rng, N, K)
    d = m.nvfp4_gemm(upload_form(a), upload_form(b), out_dtype=torch.float32).cpu().numpy()
    ref, _ = oracle.gemm_full(a, b)
    assert np.array_equal(d.astype(np.float64), ref)


@pytest.mark.parametrize("out", ["bf16", "fp32"])
def test_config1_fprop_256(out):
    # config 1: X 256x256 N(0,1) 1x16 RNE, W 256x256 N(0,0.02) 16x16 RNE, Y = X W^T
    m = nv()
    x = synth.bf16_bits(synth.activations(256, 256, seed=0))
    w = synth.bf16_bits(synth.weights(256, 256, seed=1))
    qa, qb = oracle.quantize(x), oracle.quantize(w, block=oracle.BLOCK_16x16)
    dt = torch.bfloat16 if out == "bf16" else torch.float32
    d = m.nvfp4_gemm(upload_form(qa), upload_form(qb, 1), out_dtype=dt)
    ref, sabs = oracle.gemm_full(qa, qb)
    check_gemm(bf16_to_f64(d) if out == "bf16" else d.cpu().numpy(), ref, sabs, out == "bf16", "config 1")


@pytest.mark.parametrize("M,N,K", [(512, 768, 1280), (333, 300, 416), (64, 1024, 2048)])
def test_random_ragged(M, N, K, variant):
    m = nv()
    x = synth.bf16_bits(synth.activations(M, K, seed=M))
    w = synth.bf16_bits(synth.weights(N, K, seed=N))
    qa, qb = oracle.quantize(x), oracle.quantize(w)
    d = m.nvfp4_gemm(upload_form(qa), upload_form(qb), out_dtype=torch.float32)
    ref, sabs = oracle.gemm_full(qa, qb)
    check_gemm(d.cpu().numpy(), ref, sabs, False, f"{M}x{N}x{K}")


def test_output_leading_dimension():
    m = nv()
    x = synth.bf16_bits(synth.activations(128, 256, seed=3))
    w = synth.bf16_bits(synth.weights(256, 256, seed=4))
    qa, qb = oracle.quantize(x), oracle.quantize(w)
    big = torch.full((128, 264), -7.0, dtype=torch.bfloat16, device="cuda")
    m.nvfp4_gemm(upload_form(qa), upload_form(qb), out=big[:, :256])
    ref, sabs = oracle.gemm_full(qa, qb)
    check_gemm(bf16_to_f64(big[:, :256]), ref, sabs, True, "ldd")
    assert torch.all(big[:, 256:] == -7.0)
