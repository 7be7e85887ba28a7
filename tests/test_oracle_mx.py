"""Pins of the oracle's MXFP4 quantizer, the pages' comparison format (gist.science
"Pretraining Large Language Models with NVFP4", 2.A: blocks of 32 elements, UE8M0 scale
factors, no tensor scale).  The pages give no scale rule; the oracle takes the microscaling one,
shared exponent floor(log2 amax) - 2.  The pins check it against what that rule fixes by other
means: an encoder built from numpy's frexp and ml_dtypes' E2M1 and E8M0 types, the scale's
closed form in every binade, where the block maximum lands, and the reconstruction error."""
import ml_dtypes
import numpy as np
import pytest

import synth

RNE, SR = 0, 1


def _bits(v: np.ndarray) -> np.ndarray:
    """fp32 values that are exact in bf16 -> bf16 bit patterns."""
    v = np.asarray(v, np.float32)
    b = v.view(np.uint32)
    assert np.all(b & 0xFFFF == 0), "test values must be exact in bf16"
    return (b >> 16).astype(np.uint16)


def _f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _nibbles(codes: np.ndarray) -> np.ndarray:
    r, h = codes.shape
    out = np.empty((r, 2 * h), np.uint8)
    out[:, 0::2] = codes & 15
    out[:, 1::2] = codes >> 4
    return out


def _independent_mx(v: np.ndarray):
    """The same rule through numpy/ml_dtypes: frexp for floor(log2), E8M0 and E2M1 casts."""
    rows, cols = v.shape
    blocks = v.reshape(rows, cols // 32, 32).astype(np.float64)
    amax = np.abs(blocks).max(axis=2)
    _, e2 = np.frexp(amax)
    code = np.where(amax > 0, np.clip(e2 - 1 - 2 + 127, 0, 254), 0).astype(np.int64)
    scale = np.ldexp(1.0, code - 127)
    u = np.clip(blocks / scale[:, :, None], -6.0, 6.0)           # exact: a power of two
    q = u.astype(np.float32).astype(ml_dtypes.float4_e2m1fn)
    nib = q.view(np.uint8).reshape(rows, cols) & 15
    # ml_dtypes' E8M0 agrees on the scale value (an independent decoder of the code)
    e8 = np.asarray(scale, np.float32).astype(ml_dtypes.float8_e8m0fnu).view(np.uint8)
    return nib, code.astype(np.uint8), e8


def test_scale_closed_form_every_binade(ora):
    for k in range(-133, 128):
        for m in (1.0, 1.5, 1.9921875):             # values exact in bf16 (8 significant bits)
            a = np.float32(m * 2.0 ** k)
            if a == 0 or not np.isfinite(a):
                continue
            want = min(max(k - 2 + 127, 0), 254)
            assert ora.ue8m0_of_amax(float(a)) == want, (k, m)
    assert ora.ue8m0_of_amax(0.0) == 0


@pytest.mark.parametrize("seed,scale", [(0, 1.0), (1, 1e-4), (2, 300.0)])
def test_rne_matches_independent_encoder(ora, seed, scale):
    x = synth.activations(64, 256, seed=seed, outlier_frac=0.02) if scale == 1.0 else \
        synth.grad_output(64, 256, seed=seed, std=scale)
    xb = synth.bf16_bits(x)
    codes, scales = ora.quantize_mx(xb)
    nib, code, e8 = _independent_mx(_f32(xb).reshape(xb.shape))
    assert np.array_equal(scales, code)
    assert np.array_equal(scales, e8)
    assert np.array_equal(_nibbles(codes), nib)


def test_block_maximum_lands_in_the_top_binade(ora):
    # amax / 2^E is in [4, 8): RNE gives 4 for [4, 5], 6 above 5 (5 is a tie, to the even code 4)
    rng = np.random.default_rng(3)
    v = rng.standard_normal((32, 128)).astype(np.float32)
    v = np.ascontiguousarray((v.view(np.uint32) & 0xFFFF0000).view(np.float32))   # exact in bf16
    codes, scales = ora.quantize_mx(_bits(v))
    nib = _nibbles(codes)
    blocks = v.reshape(32, 4, 32)
    for r in range(32):
        for b in range(4):
            j = int(np.argmax(np.abs(blocks[r, b])))
            u = abs(float(blocks[r, b, j])) / 2.0 ** (int(scales[r, b]) - 127)
            assert 4.0 <= u < 8.0
            assert (nib[r, b * 32 + j] & 7) == (6 if u <= 5.0 else 7)


def test_reconstruction_bound(ora):
    # decoded with ml_dtypes: |v - q 2^E| <= half a step of E2M1 (0.25, 0.5 or 1 times 2^E by
    # binade), or the saturation gap |v| - 6 * 2^E above the grid
    x = synth.activations(128, 512, seed=5, outlier_frac=0.01)
    xb = synth.bf16_bits(x)
    codes, scales = ora.quantize_mx(xb)
    v = _f32(xb).astype(np.float64).reshape(128, 512)
    q = _nibbles(codes).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    s = scales.view(ml_dtypes.float8_e8m0fnu).astype(np.float64).repeat(32, axis=1)
    err = np.abs(v - q * s)
    u = np.abs(v) / s
    half = np.select([u < 2, u < 4], [0.25, 0.5], 1.0) * s
    bound = np.where(u > 6, np.abs(v) - 6 * s, half)
    assert np.all(err <= bound * (1 + 1e-12) + 1e-300)


def test_sr_unbiased_per_element(ora):
    # one block repeated over many rows: each row draws its own Philox fields, so the mean of the
    # decoded values converges to v (SR is unbiased below the saturation point)
    # block amax 2.55: E = floor(log2 2.55) - 2 = -1, so u = 2 v and every |u| <= 5.1 < 6
    vals = np.array([0.15, -0.85, 1.3, 0.025, -2.2, 2.55, 0.5, -0.45] * 4, np.float32)
    vals = np.ascontiguousarray((vals.view(np.uint32) & 0xFFFF0000).view(np.float32))   # exact in bf16
    rows = 20000
    x = np.tile(_bits(vals), (rows, 1))
    codes, scales = ora.quantize_mx(x, mode=SR, sr_seed=11, stream_id=2)
    q = _nibbles(codes).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    s = scales.view(ml_dtypes.float8_e8m0fnu).astype(np.float64).repeat(32, axis=1)
    mean = (q * s).mean(axis=0)
    sd = (q * s).std(axis=0) / np.sqrt(rows) + 1e-12
    assert np.all(np.abs(mean - vals.astype(np.float64)) <= 4 * sd + 2.0 ** -16 * np.abs(vals))


def test_hand_worked_block(ora):
    # amax 3 -> floor(log2 3) = 1 -> E = -1, scale code 126, u = 2 v:
    #   3.0 -> u = 6 -> code 7;   -1.25 -> u = -2.5, a tie between 2 and 3 -> the even code 4
    #   (value 2), sign -> 0xC;   bf16(0.6) = 0.6015625 -> u = 1.203 -> nearest 1 -> code 2;
    #   bf16(0.1) = 0.10009765625 -> u = 0.2002 < 0.25 -> 0;   zeros -> 0
    v = np.zeros(32, np.float32)
    v[:4] = [3.0, -1.25, 0.6015625, 0.10009765625]
    codes, scales = ora.quantize_mx(_bits(v)[None, :])
    assert scales.tolist() == [[126]]
    assert codes[0, 0] == 0xC7 and codes[0, 1] == 0x02 and not codes[0, 2:].any()


def test_mx_dequantize_and_gemm_match_independent_decoder(ora):
    # the oracle's MXFP4 dequantizer and fp64 GEMM against ml_dtypes' E2M1 and E8M0 decoders
    import ml_dtypes
    x = synth.bf16_bits(synth.activations(48, 256, seed=3, outlier_frac=0.05))
    w = synth.bf16_bits(synth.weights(40, 256, seed=4))
    (ca, sa), (cb, sb) = ora.quantize_mx(x), ora.quantize_mx(w, mode=SR, sr_seed=5, stream_id=1)

    def ml(codes, scales):
        nib = np.empty((codes.shape[0], codes.shape[1] * 2), np.uint8)
        nib[:, 0::2], nib[:, 1::2] = codes & 15, codes >> 4
        vals = nib.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
        return vals * scales.view(ml_dtypes.float8_e8m0fnu).astype(np.float64).repeat(32, axis=1)

    A, B = ml(ca, sa), ml(cb, sb)
    assert np.array_equal(ora.dequantize_mx(ca, sa), A)
    d, s = ora.gemm_mx(ca, sa, cb, sb)
    ref = A @ B.T
    assert np.allclose(d, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    assert np.allclose(s, np.abs(A) @ np.abs(B).T, rtol=1e-12)


def test_mx_swizzle_places_every_scale_once(ora):
    # the tile layout is a bijection from (row, block) onto the non-padding bytes: tag every
    # scale with a distinct value and read each back at its closed-form offset
    R, K = 200, 96 * 4
    sc = (np.arange(R * (K // 32)) % 251 + 1).astype(np.uint8).reshape(R, K // 32)
    sw = ora.mx_scales_swizzled(sc, K)
    nkt = (K // 32 + 3) // 4
    rr, kk = np.meshgrid(np.arange(R), np.arange(K // 32), indexing="ij")
    off = ((rr // 128) * nkt + kk // 4) * 512 + (rr % 32) * 16 + ((rr // 32) % 4) * 4 + kk % 4
    assert np.array_equal(sw[off], sc)
    assert np.count_nonzero(sw) == sc.size
