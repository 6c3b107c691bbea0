"""Pins of the oracle's RMS normalisation, the element-wise operator taken to
precede a layer whose table precompute is fused into it (LUT Tensor Core
notes, Section 3.1.1: the precompute fused with the preceding element-wise
operator; the operator read as the RMSNorm of a LLaMA-style block,
x = h * gamma / sqrt(mean(h^2) + eps)).

  * hand-computed values, with and without eps and with a non-unit gamma;
  * invariants: with eps = 0 the result does not change when h is scaled by
    any s > 0, and x / gamma has mean square 1; with eps > 0, x / (h gamma)
    is the constant 1 / sqrt(mean(h^2) + eps); h = 0 gives x = 0.
Planted mistakes (a sum in place of the mean, eps added outside the square
root, gamma dropped) each fail a pin.
"""
import math

import numpy as np
import pytest

import oracle


def pin_rmsnorm(f):
    # hand-computed: h = (3, 4): mean(h^2) = 12.5
    x = f(np.array([3.0, 4.0]), np.array([1.0, 1.0]), 0.0)
    assert np.allclose(x, [3 / math.sqrt(12.5), 4 / math.sqrt(12.5)], rtol=1e-15, atol=0)
    x = f(np.array([3.0, 4.0]), np.array([2.0, -1.0]), 0.5)
    assert np.allclose(x, [6 / math.sqrt(13.0), -4 / math.sqrt(13.0)], rtol=1e-15, atol=0)
    g = np.random.default_rng(3)
    for n in (1, 7, 4096):
        h = g.standard_normal(n) * 10.0 ** g.integers(-2, 3)
        gam = g.uniform(0.5, 2.0, n)
        base = f(h, gam, 0.0)
        for s in (0.25, 3.0, 1e3):
            assert np.allclose(f(s * h, gam, 0.0), base, rtol=1e-13, atol=0)
        assert abs(np.mean((base / gam) ** 2) - 1.0) < 1e-12
        eps = 0.37
        want = 1.0 / math.sqrt(np.mean(h * h) + eps)
        assert np.allclose(f(h, gam, eps) / (h * gam), want, rtol=1e-13, atol=0)
    assert np.all(f(np.zeros(5), np.ones(5), 1e-6) == 0.0)


def test_oracle_rmsnorm_pins():
    pin_rmsnorm(oracle.rmsnorm)


def test_oracle_linear_rmsnorm_is_linear_of_normalised_row():
    from lut_binary_basis_b200.synth import LayerSpec, make_layer
    spec = LayerSpec("n", 7, 24, 2, 1, 5, 8)
    layer = make_layer(spec, [91])
    h = np.random.default_rng(92).standard_normal(24)
    gam = np.random.default_rng(93).uniform(0.5, 1.5, 24)
    x = oracle.rmsnorm(h, gam, 1e-5)
    assert np.array_equal(oracle.linear_rmsnorm(layer, h, gam, 1e-5), oracle.linear(layer, x[None, :]))


def _sum_not_mean(h, gamma, eps):
    h = np.asarray(h, np.float64)
    return h * gamma / np.sqrt(np.sum(h * h) + eps)


def _eps_outside(h, gamma, eps):
    h = np.asarray(h, np.float64)
    return h * gamma / (np.sqrt(np.mean(h * h)) + eps)


def _no_gamma(h, gamma, eps):
    h = np.asarray(h, np.float64)
    return h / np.sqrt(np.mean(h * h) + eps)


@pytest.mark.parametrize("broken", [_sum_not_mean, _eps_outside, _no_gamma],
                         ids=["sum_not_mean", "eps_outside_sqrt", "gamma_dropped"])
def test_planted_rmsnorm_mistake_is_caught(broken):
    with pytest.raises(AssertionError):
        pin_rmsnorm(broken)
