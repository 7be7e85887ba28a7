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
