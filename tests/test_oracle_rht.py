"""Pins of the oracle's 16-point Random Hadamard Transform.

gist.science "Pretraining Large Language Models with NVFP4", Technische Zusammenfassung 2.B.2:
outliers are spread by multiplying with Hadamard matrices (an orthogonal rotation); 16x16 is
the size used; applied to the Wgrad inputs.  The oracle computes 0.25 * H16 * (D x) with a
fixed butterfly.  The pins: the closed-form Sylvester matrix H[i][j] = (-1)^popcount(i & j)
evaluated in fp64, orthogonality, the exact one-hot response and the inverse round trip.
"""
import numpy as np
import pytest

H16 = np.array([[(-1) ** bin(i & j).count("1") for j in range(16)] for i in range(16)], np.float64)


def test_sylvester_closed_form_is_orthogonal():
    assert np.array_equal(H16 @ H16.T, 16 * np.eye(16))


@pytest.mark.parametrize("seed", [0, 1, 7, 12345])
def test_butterfly_matches_closed_form(ora, seed):
    rng = np.random.default_rng(seed)
    signs = ora.rht_signs(seed)
    d = np.array([-1.0 if (signs >> j) & 1 else 1.0 for j in range(16)])
    for _ in range(200):
        x = rng.standard_normal(16).astype(np.float32) * np.float32(rng.choice([1e-3, 1.0, 50.0]))
        got = ora.rht16(x, signs).astype(np.float64)
        want = 0.25 * H16 @ (d * x.astype(np.float64))
        assert np.allclose(got, want, rtol=0, atol=1e-6 * np.abs(x).sum())


def test_one_hot_response_is_exactly_quarter(ora):
    for seed in (0, 3):
        signs = ora.rht_signs(seed)
        for j in range(16):
            e = np.zeros(16, np.float32)
            e[j] = 1.0
            got = ora.rht16(e, signs)
            sj = -1.0 if (signs >> j) & 1 else 1.0
            assert np.array_equal(got, (0.25 * sj * H16[:, j]).astype(np.float32))


def test_round_trip_is_identity(ora):
    rng = np.random.default_rng(5)
    signs = ora.rht_signs(11)
    d = np.array([-1.0 if (signs >> j) & 1 else 1.0 for j in range(16)])
    for _ in range(100):
        x = rng.standard_normal(16).astype(np.float32)
        y = ora.rht16(x, signs).astype(np.float64)
        # Q = 0.25 H D is orthogonal: Q^T Q = D H^T H D / 16 = I, so x = D (0.25 H^T) y
        back = d * (H16.T @ y) * 0.25
        assert np.allclose(back, x, rtol=0, atol=1e-6)


def test_signs_depend_on_seed(ora):
    s = {ora.rht_signs(seed) for seed in range(64)}
    assert len(s) > 50
    assert all(0 <= v < (1 << 16) for v in s)


def test_every_sign_bit_is_a_fair_coin_over_seeds(ora):
    # The pages call the rotation "random": each of the 16 diagonal signs must be +1 or -1 with
    # probability 1/2 over seeds.  Over 10^4 seeds every bit's frequency lies within 4 sigma of
    # 1/2 (sigma = 0.005), every pair of bits agrees about half the time, and the 16-bit words
    # are nearly all distinct (a mask that kept 8 of the 16 bits, a stuck bit, or one word shared
    # by both halves fails one of these).
    n = 10000
    words = np.array([ora.rht_signs(seed) for seed in range(n)], np.uint32)
    bits = ((words[:, None] >> np.arange(16)) & 1).astype(np.float64)
    freq = bits.mean(axis=0)
    assert np.all(np.abs(freq - 0.5) < 4 * 0.005), freq
    agree = (bits[:, :, None] == bits[:, None, :]).mean(axis=0)
    off = agree[~np.eye(16, dtype=bool)]
    assert np.all(np.abs(off - 0.5) < 4 * 0.005), off.min()
    # 10^4 draws from 2^16 values: about 9.3e3 distinct in expectation
    assert len(set(words.tolist())) > 9000


@pytest.mark.parametrize("seed", [0, 5, 2 ** 40 + 3])
def test_quantizer_rotates_with_the_signs_of_its_seed(ora, seed):
    # The RHT form of a column holding one nonzero value e_j in a 16-token group has, in its
    # 16 outputs, exactly 0.25 * s_j * H[:, j] times that value: the sign the quantizer applied
    # to token j is read back from its codes and equals bit j of rht_signs(seed).
    signs = ora.rht_signs(seed)
    for j in range(16):
        x = np.zeros((16, 16), np.uint16)
        x[j, 0] = 0x3F80          # bf16 1.0 in column 0 at token j
        q = ora.quantize(x, along=1, rht=True, rht_seed=seed)
        nib = q.nibbles()[0]      # form row 0 = source column 0, K = the 16 tokens
        # every output has magnitude 0.25 -> the block maximum, code 6.0 (0x7) with its sign
        assert np.all((nib & 7) == 7), nib
        got_sign = np.where(nib & 8, -1.0, 1.0)
        sj = -1.0 if (signs >> j) & 1 else 1.0
        assert np.array_equal(got_sign, sj * H16[:, j]), (j, got_sign)
