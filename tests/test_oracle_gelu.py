"""Pins of the oracle's GeLU glue of the one-FFN training step (erf form, bf16 in and out).

The activation is not part of the pages' method; the FFN step of the workload needs it between
the up- and down-projections.  The oracle evaluates g = h * Phi(h) and dh = dg * (Phi(h) +
h * phi(h)) in fp64 and rounds to bf16 (through fp32).  The pins compare it with an independent
normal CDF (scipy.special.ndtr), the closed-form values at 0, the odd-part identity
g(h) - g(-h) = h, and central finite differences of the forward for the backward."""
import numpy as np
import pytest
import torch
from scipy.special import ndtr


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp64 -> fp32 (RNE) -> bf16 (RNE), as bit patterns: the oracle's rounding chain."""
    t = torch.from_numpy(np.asarray(x, np.float64).astype(np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _inputs():
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.1, 1.0, 3.0)] +
                       [np.array([0.0, -0.0, 1.0, -1.0, 2.0, -2.0, 5.0, -5.0, 10.0, -10.0, 40.0, -40.0, 1e-30])])
    return _bf16_bits(x)


def _ulps(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in bf16 steps between bit patterns (sign-magnitude to a monotone integer line)."""
    def line(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)
    return np.abs(line(a_bits) - line(b_bits))


def test_forward_against_independent_cdf(ora):
    h = _inputs()
    g = ora.gelu_fwd(h)
    ref = _bf16_bits(_f64(h) * ndtr(_f64(h)))
    # both round the same fp64 value: equal except where the two CDFs differ across a rounding
    # boundary, which moves the result by at most one bf16 step
    d = _ulps(g, ref)
    assert d.max() <= 1
    assert np.mean(d == 0) > 0.999


def test_forward_closed_forms(ora):
    pts = _bf16_bits(np.array([0.0, 1.0, -1.0, 40.0, -40.0]))
    g = _f64(ora.gelu_fwd(pts))
    assert g[0] == 0.0
    assert g[1] == _f64(_bf16_bits(np.array([0.8413447460685429])))[0]      # Phi(1)
    assert g[2] == _f64(_bf16_bits(np.array([-0.15865525393145707])))[0]    # -(1 - Phi(1))
    assert g[3] == 40.0 and g[4] == 0.0


def test_forward_odd_part_is_identity(ora):
    # g(h) - g(-h) = h * (Phi(h) + Phi(-h) - 1 + 1) = h, up to the two bf16 roundings
    h = _inputs()
    h = h[np.abs(_f64(h)) > 1e-3]
    neg = h ^ np.uint16(0x8000)
    lhs = _f64(ora.gelu_fwd(h)) - _f64(ora.gelu_fwd(neg))
    x = _f64(h)
    tol = 2.0 ** -8 * (np.abs(x) * ndtr(np.abs(x)) + np.abs(x) * ndtr(-np.abs(x))) * 1.01 + 1e-300
    assert np.all(np.abs(lhs - x) <= tol)


def test_backward_is_derivative_of_forward(ora):
    rng = np.random.default_rng(11)
    x = _bf16_bits(rng.standard_normal(5000) * 2.0)
    xs = _f64(x)
    one = _bf16_bits(np.ones_like(xs))
    dh = _f64(ora.gelu_bwd(x, one))
    eps = 1e-6
    fd = ((xs + eps) * ndtr(xs + eps) - (xs - eps) * ndtr(xs - eps)) / (2 * eps)
    # bf16 output: half a step relative, plus the finite-difference error (~1e-10)
    assert np.all(np.abs(dh - fd) <= 2.0 ** -8 * np.abs(fd) + 1e-8)
    # GeLU'(0) = Phi(0) = 1/2 exactly
    z = _bf16_bits(np.array([0.0]))
    assert _f64(ora.gelu_bwd(z, _bf16_bits(np.array([1.0]))))[0] == 0.5


@pytest.mark.parametrize("scale", [1e-4, 1.0])
def test_backward_is_linear_in_dg(ora, scale):
    # dh = dg * GeLU'(h): doubling dg (exact in bf16) doubles dh exactly
    rng = np.random.default_rng(3)
    h = _bf16_bits(rng.standard_normal(4000))
    dg = _bf16_bits(rng.standard_normal(4000) * scale)
    dg2 = _bf16_bits(_f64(dg) * 2.0)
    assert np.array_equal(_f64(ora.gelu_bwd(h, dg2)), 2.0 * _f64(ora.gelu_bwd(h, dg)))
