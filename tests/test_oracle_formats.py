"""Pins of the oracle's number formats against an independent implementation (ml_dtypes).

E2M1 and E4M3 come from the NVFP4 format description (gist.science "Pretraining Large Language
Models with NVFP4", Technische Zusammenfassung 2.A): 4-bit floating-point elements with an E4M3
scale per 16-element block.  ml_dtypes implements both OCP formats with round-to-nearest-even;
its E4M3 returns NaN instead of saturating above ~464, so inputs are clamped to 448 first.
"""
import ml_dtypes
import numpy as np
import pytest


def _floats_with_exponent(e: int, sign: int) -> np.ndarray:
    """Every fp32 with unbiased exponent e (all 2^23 mantissas) and the given sign."""
    m = np.arange(1 << 23, dtype=np.uint32)
    bits = (np.uint32(sign) << np.uint32(31)) | (np.uint32(e + 127) << np.uint32(23)) | m
    return bits.view(np.float32)


def _ml_e2m1_codes(x: np.ndarray) -> np.ndarray:
    return x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF


def test_e2m1_value_set(ora):
    vals = [ora.e2m1_value(c) for c in range(16)]
    assert vals[:8] == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert vals[8:] == [-0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]
    ref = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(np.array(vals), ref)


@pytest.mark.parametrize("e", [-3, -2, -1, 0, 1, 2])
@pytest.mark.parametrize("sign", [0, 1])
def test_e2m1_rne_exhaustive_decision_range(ora, e, sign):
    # every fp32 in [2^e, 2^(e+1)): all of E2M1's rounding midpoints (0.25 .. 5) and its
    # saturation point 6 fall inside e = -3 .. 2
    x = _floats_with_exponent(e, sign)
    got = ora.e2m1_rne(x)
    want = _ml_e2m1_codes(x)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"first mismatch x={x[bad[0]]!r} oracle={got[bad[0]]} ml_dtypes={want[bad[0]]}"


def test_e2m1_rne_random_patterns(ora):
    rng = np.random.default_rng(1234)
    bits = rng.integers(0, 1 << 32, size=4_000_000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    assert np.array_equal(ora.e2m1_rne(x), _ml_e2m1_codes(x))


def test_e2m1_rne_special_cases(ora):
    x = np.array([0.0, -0.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 6.5, 1e30, np.inf, -np.inf,
                  -0.1, 1e-45, -1e-45], np.float32)
    want = [0x0, 0x8, 0x0, 0x2, 0x2, 0x4, 0x4, 0x6, 0x6, 0x7, 0x7, 0x7, 0x7, 0xF, 0x8, 0x0, 0x8]
    assert list(ora.e2m1_rne(x)) == want


def test_e4m3_decode_all_codes(ora):
    ours = np.array([ora.e4m3_value(c) for c in range(256)])
    ref = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert ora.e4m3_value(0x7E) == 448.0 and ora.e4m3_value(0x01) == 2.0 ** -9


def _ml_e4m3_codes(x: np.ndarray) -> np.ndarray:
    return np.minimum(x, np.float32(448.0)).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)


def test_e4m3_rne_sat_near_every_boundary(ora):
    # the encoder is piecewise constant; its decisions sit at the midpoints between adjacent
    # codes.  Check every fp32 within +-4096 ulp of each midpoint and of each code value.
    vals = np.array([ora.e4m3_value(c) for c in range(0x7F)], np.float64)
    points = np.concatenate([vals, (vals[:-1] + vals[1:]) / 2, [448.0, 464.0, 480.0]]).astype(np.float32)
    points = points[points > 0]
    offs = np.arange(-4096, 4097, dtype=np.int64)
    bits = (points.view(np.uint32).astype(np.int64)[:, None] + offs[None, :]).reshape(-1)
    bits = bits[(bits > 0) & (bits < 0x7F800000)].astype(np.uint32)
    x = bits.view(np.float32)
    got = ora.e4m3_rne_sat(x)
    want = _ml_e4m3_codes(x)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"x={x[bad[0]]!r} oracle={got[bad[0]]:#x} ml_dtypes={want[bad[0]]:#x}"


def test_e4m3_rne_sat_random_and_saturation(ora):
    rng = np.random.default_rng(99)
    x = rng.uniform(0, 1, 2_000_000).astype(np.float32) * np.float32(2.0) ** rng.integers(-30, 20, 2_000_000).astype(np.float32)
    got = ora.e4m3_rne_sat(x)
    assert np.array_equal(got, _ml_e4m3_codes(x))
    big = np.array([448.0, 449.0, 464.0, 465.0, 1e6, np.inf], np.float32)
    assert list(ora.e4m3_rne_sat(big)) == [0x7E] * 6
    assert list(ora.e4m3_rne_sat(np.array([0.0, 2.0 ** -10, 2.0 ** -10 * 1.0001, 2.0 ** -9], np.float32))) == [0, 0, 1, 1]
