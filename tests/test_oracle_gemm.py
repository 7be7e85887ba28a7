"""Pins of the oracle's fp64 block-scaled GEMM D = A * B^T.

brainai.pro "NVFP4 Entraine en precision 16 bits ...", Details techniques: the FP4 GEMMs of the
fully-connected layers carry the training time; gist.science "Pretraining Large Language Models
with NVFP4", 3 (Beitraege): Blackwell tensor cores run FP4.  The oracle dequantizes with its own
tables; the pins decode the same bytes through ml_dtypes (an independent decoder) and multiply
with numpy.
"""
import ml_dtypes
import numpy as np

import synth


def _ml_dequant(q):
    nib = q.nibbles()
    vals = nib.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    sc = q.scales_rm.view(ml_dtypes.float8_e4m3fn).astype(np.float64).repeat(16, axis=1)
    return vals * sc * np.float64(q.s_t)


def test_dequantize_matches_independent_decoder(ora):
    x = synth.bf16_bits(synth.activations(64, 128, seed=1, outlier_frac=0.02))
    q = ora.quantize(x)
    assert np.array_equal(q.dequantize(), _ml_dequant(q))


def test_gemm_full_matches_numpy(ora):
    a = ora.quantize(synth.bf16_bits(synth.activations(96, 256, seed=2)))
    b = ora.quantize(synth.bf16_bits(synth.weights(80, 256, seed=3)), block=ora.BLOCK_16x16)
    d, s = ora.gemm_full(a, b)
    A, B = _ml_dequant(a), _ml_dequant(b)
    ref = A @ B.T
    assert np.allclose(d, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    assert np.allclose(s, np.abs(A) @ np.abs(B).T, rtol=1e-12)


def test_gemm_small_integers_exact(ora):
    # operands built directly from random codes, power-of-two block scales and a power-of-two
    # tensor scale: every product and every partial sum is a short dyadic number, so the
    # oracle and an independent numpy evaluation must agree exactly
    rng = np.random.default_rng(0)
    pow2_codes = np.array([0x38, 0x40, 0x48, 0x30, 0x28], np.uint8)   # 1, 2, 4, 0.5, 0.25
    for M, N, K in ((8, 8, 16), (16, 8, 32), (4, 12, 64)):
        def make(R):
            nib = rng.integers(0, 16, size=(R, K), dtype=np.uint8)
            codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
            sc = rng.choice(pow2_codes, size=(R, K // 16))
            return ora.QForm(R, K, np.ascontiguousarray(codes), np.ascontiguousarray(sc), None, None, 1.0,
                             float(np.float32(0.125)))
        a, b = make(M), make(N)
        d, _ = ora.gemm_full(a, b)
        assert np.array_equal(d, _ml_dequant(a) @ _ml_dequant(b).T)


def test_sampled_equals_full(ora):
    a = ora.quantize(synth.bf16_bits(synth.activations(130, 96, seed=5)))
    b = ora.quantize(synth.bf16_bits(synth.weights(70, 96, seed=6)))
    d, s = ora.gemm_full(a, b)
    ii, jj = synth.sample_indices(130, 70, 500, seed=1)
    ds, ss = ora.gemm_sampled(a, b, ii, jj, nthreads=3)
    assert np.array_equal(ds, d[ii, jj]) and np.array_equal(ss, s[ii, jj])


def test_rht_cancels_in_wgrad(ora):
    # the same random-sign Hadamard rotation on both wgrad operands along K cancels:
    # sum_t (Q dy)(Q x) = sum_t dy x up to the quantization error; without quantization
    # (checked on the fp32 transformed values) it is exact to fp32 rounding
    T, n, d = 64, 32, 48
    dy = synth.bf16_bits(synth.grad_output(T, n, seed=2))
    x = synth.bf16_bits(synth.activations(T, d, seed=0))
    signs = ora.rht_signs(9)
    f = lambda m: ora.bf16_bits_to_f32(m).reshape(m.shape).astype(np.float32)
    def rot(m):
        mt = f(m).T
        return np.stack([np.concatenate([ora.rht16(r[k:k + 16], signs) for k in range(0, T, 16)]) for r in mt])
    ref = f(dy).T.astype(np.float64) @ f(x).astype(np.float64)
    got = rot(dy).astype(np.float64) @ rot(x).astype(np.float64).T
    assert np.allclose(got, ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max())


def test_bf16_gemm_is_the_exact_product(ora):
    # the BF16 path's oracle GEMM: integer-valued bf16 operands make every product and sum an exact
    # integer, checked against Python's arbitrary-precision integers; a fractional case against
    # Fraction arithmetic on the decoded bf16 values
    from fractions import Fraction
    import torch
    g = torch.Generator().manual_seed(3)
    a = torch.randint(-64, 65, (7, 40), generator=g).to(torch.bfloat16)
    b = torch.randint(-64, 65, (5, 40), generator=g).to(torch.bfloat16)
    d, s = ora.gemm_bf16(synth.bf16_bits(a), synth.bf16_bits(b))
    ai, bi = a.to(torch.int64).tolist(), b.to(torch.int64).tolist()
    for i in range(7):
        for j in range(5):
            assert d[i, j] == sum(x * y for x, y in zip(ai[i], bi[j]))
            assert s[i, j] == sum(abs(x * y) for x, y in zip(ai[i], bi[j]))
    x = (torch.randn(3, 24, generator=g) * 3).to(torch.bfloat16)
    w = (torch.randn(4, 24, generator=g) * 0.02).to(torch.bfloat16)
    d, _ = ora.gemm_bf16(synth.bf16_bits(x), synth.bf16_bits(w))
    xf = [[Fraction(float(v)) for v in row] for row in x.float().tolist()]
    wf = [[Fraction(float(v)) for v in row] for row in w.float().tolist()]
    for i in range(3):
        for j in range(4):
            exact = sum(p * q for p, q in zip(xf[i], wf[j]))
            assert abs(Fraction(d[i, j]) - exact) <= abs(exact) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 80)
