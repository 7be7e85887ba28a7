"""Pins of the oracle's stochastic rounding and its Philox4x32-10 bit source.

gist.science "Pretraining Large Language Models with NVFP4", Technische Zusammenfassung 2.B.4:
gradients are rounded stochastically -- to one of the two nearest representable values with a
probability that removes the bias.  The pins are statistical (unbiasedness, frequency of the
upward choice at 3 sigma over 1e6 draws), exactness of representable values, and the closed
form of the threshold for dyadic fractions.

Philox parity: numpy's Philox is the 4x64 variant and no known-answer file is in the image, so
on the CPU the generator is pinned only by uniformity and independence statistics; the exact
pin is the GPU test against cuRAND's Philox4_32_10 (tests/test_gpu_philox_curand.py).
"""
import numpy as np
import pytest

GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _decode(codes):
    mag = np.array(GRID)[codes & 7]
    return np.where(codes & 8, -mag, mag)


@pytest.mark.parametrize("u", [0.1, 0.3, 0.6, 1.2, 1.7, 2.4, 2.9, 3.3, 4.5, 5.9, -0.2, -2.2, -5.5])
def test_sr_unbiased(ora, u):
    n = 1_000_000
    idx = np.arange(n, dtype=np.uint64) + np.uint64(12_345_678)
    r = ora.sr_bits16(seed=42, stream_id=1, idx=idx)
    codes = ora.e2m1_sr(np.full(n, u, np.float32), r)
    vals = _decode(codes)
    a = abs(u)
    lo = max(g for g in GRID if g <= a)
    hi = min(g for g in GRID if g > a)
    step = hi - lo
    f = (a - lo) / step
    # only the two neighbours may appear
    assert set(np.unique(np.abs(vals))) <= {lo, hi}
    p_up = np.mean(np.abs(vals) == hi)
    sigma_p = np.sqrt(f * (1 - f) / n)
    assert abs(p_up - f) <= 3 * sigma_p + 2.0 ** -16
    sigma_mean = step * sigma_p
    assert abs(vals.mean() - np.float32(u)) <= 3 * sigma_mean + step * 2.0 ** -16


def test_sr_representable_values_never_move(ora):
    n = 200_000
    r = ora.sr_bits16(7, 2, np.arange(n, dtype=np.uint64))
    for g in GRID:
        for s in (1.0, -1.0):
            codes = ora.e2m1_sr(np.full(n, s * g, np.float32), r)
            want = ora.e2m1_rne(np.array([s * g], np.float32))[0]
            assert np.all(codes == want)


def test_sr_threshold_closed_form(ora):
    # for u = lo + f*step with f = m / 2^16 exactly, the threshold is m
    for lo, hi in zip(GRID[:-1], GRID[1:]):
        for m in (0, 1, 2, 255, 32768, 65535):
            u = np.float32(lo + (hi - lo) * m / 65536.0)
            assert ora.e2m1_sr_threshold(np.array([u]))[0] == m
    # above the grid: saturation, never rounds
    assert ora.e2m1_sr_threshold(np.array([6.0, 7.0, np.inf], np.float32)).tolist() == [0, 0, 0]


def test_sr_saturates_and_keeps_sign(ora):
    r = np.array([0, 65535, 12345], np.uint32)
    assert ora.e2m1_sr(np.array([6.5, -7.0, 1e9], np.float32), r).tolist() == [7, 15, 7]
    assert ora.e2m1_sr(np.array([-0.0, 0.0], np.float32), np.array([0, 0], np.uint32)).tolist() == [8, 0]


def test_philox_fields_uniform(ora):
    n = 1 << 20
    r = ora.sr_bits16(2024, 1, np.arange(n, dtype=np.uint64))
    assert r.max() < 65536
    # chi-square over 256 bins of the top byte
    hist = np.bincount((r >> 8).astype(np.int64), minlength=256)
    expected = n / 256
    chi2 = ((hist - expected) ** 2 / expected).sum()
    assert chi2 < 255 + 6 * np.sqrt(2 * 255)
    # every bit balanced
    for b in range(16):
        p = ((r >> b) & 1).mean()
        assert abs(p - 0.5) < 4 * 0.5 / np.sqrt(n)


def test_philox_streams_and_seeds_independent(ora):
    n = 1 << 18
    idx = np.arange(n, dtype=np.uint64)
    a = ora.sr_bits16(1, 1, idx).astype(np.float64)
    b = ora.sr_bits16(1, 2, idx).astype(np.float64)
    c = ora.sr_bits16(2, 1, idx).astype(np.float64)
    for u, v in ((a, b), (a, c)):
        corr = np.corrcoef(u, v)[0, 1]
        assert abs(corr) < 5 / np.sqrt(n)
        assert np.mean(u == v) < 0.001


def test_philox_counter_layout(ora):
    # the 16-bit field of element i is field (i mod 8) of the block for counter g = i // 8
    blocks = ora.philox_blocks(seed=0xDEADBEEF12345678, stream_id=3, g0=1000, n=4)
    idx = np.arange(8000, 8032, dtype=np.uint64)
    r = ora.sr_bits16(0xDEADBEEF12345678, 3, idx)
    for t in range(32):
        w = blocks[t // 8][(t % 8) // 2]
        assert r[t] == (int(w) >> (16 * (t % 2))) & 0xFFFF
    # reproducible
    assert np.array_equal(r, ora.sr_bits16(0xDEADBEEF12345678, 3, idx))
