"""Pins of the SmoothQuant comparator oracle (per-channel scaling, then MXFP4) against
what the mathematics fixes: special cases that reduce to the plain encoder, exact
power-of-two behaviour, the migration balance of the scale rule, the smoothing identity
and brute force."""
import numpy as np
import pytest

from oracle import mxfp4
from oracle import smoothquant as sq


def _x(seed, M=8, K=96):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K)).astype(np.float32) * rng.uniform(0.1, 20, K).astype(np.float32)
    return X.astype(np.float64)


def test_unit_scale_is_plain_encoder():
    X = _x(0)
    act = sq.quantize_act(X, np.ones(X.shape[1], np.float32))
    c, s = mxfp4.encode(X)
    np.testing.assert_array_equal(act["codes"], c)
    np.testing.assert_array_equal(act["scales"], s)


@pytest.mark.parametrize("k", [-5, -1, 3])
def test_power_of_two_scale_shifts_only_the_exponent(k):
    """A common power-of-two inverse scale on a whole block multiplies every value
    exactly, so the codes are unchanged and each scale byte moves by k."""
    X = _x(1)
    inv = np.full(X.shape[1], 2.0 ** k, np.float32)
    act = sq.quantize_act(X, inv)
    c, s = mxfp4.encode(X)
    np.testing.assert_array_equal(act["codes"], c)
    np.testing.assert_array_equal(act["scales"].astype(int), s.astype(int) + k)


def test_migration_balance_alpha_half():
    """s_j = sqrt(max|X_j| / max|W_j|) makes the channel maxima of X/s and sW equal."""
    rng = np.random.default_rng(2)
    X = _x(2, M=16, K=64)
    W = rng.standard_normal((64, 40)) * rng.uniform(0.01, 1, (64, 1))
    s = sq.scales_from(X, W, alpha=0.5)
    xm = np.abs(X / s[None, :]).max(axis=0)
    wm = np.abs(sq.smooth_weight(W, s)).max(axis=1)
    np.testing.assert_allclose(xm, wm, rtol=1e-12)


def test_alpha_limits():
    rng = np.random.default_rng(3)
    X = _x(3, M=16, K=32)
    W = rng.standard_normal((32, 8))
    s1 = sq.scales_from(X, W, alpha=1.0)           # all of the range moves to the weight
    np.testing.assert_allclose(np.abs(X / s1).max(axis=0), 1.0, rtol=1e-12)
    s0 = sq.scales_from(X, W, alpha=0.0)           # none of it: weight channels become unit
    np.testing.assert_allclose(np.abs(sq.smooth_weight(W, s0)).max(axis=1), 1.0, rtol=1e-12)


def test_zero_channel_gets_unit_scale():
    s = sq.smooth_scales(np.array([0.0, 4.0, 2.0]), np.array([1.0, 0.0, 0.5]))
    np.testing.assert_array_equal(s, [1.0, 1.0, 2.0])


def test_smoothing_identity():
    rng = np.random.default_rng(4)
    X = _x(4, M=12, K=64)
    W = rng.standard_normal((64, 24))
    s = sq.scales_from(X, W)
    lhs = (X / s[None, :]) @ sq.smooth_weight(W, s)
    np.testing.assert_allclose(lhs, X @ W, rtol=1e-12, atol=1e-12)


def test_scaled_values_match_bruteforce_encoder():
    X = _x(5, M=6, K=64)
    inv = sq.inverse_scales_f32(np.random.default_rng(5).uniform(0.05, 30, 64))
    act = sq.quantize_act(X, inv)
    c, s = mxfp4.encode_bruteforce(act["Xs"])
    np.testing.assert_array_equal(act["codes"], c)
    np.testing.assert_array_equal(act["scales"], s)
    # the product is the float32 product, nothing finer
    np.testing.assert_array_equal(act["Xs"], (X.astype(np.float32) * inv).astype(np.float64))


def test_lossless_case():
    """Activations and smoothed weights on the E2M1 grid times one power of two per
    block: quantization is exact and Y equals X W."""
    rng = np.random.default_rng(6)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    M, K, N = 4, 64, 8
    X = rng.choice(grid, (M, K)) * rng.choice([-1, 1], (M, K))
    W = rng.choice(grid, (K, N)) * rng.choice([-1, 1], (K, N)) / 4
    s = np.ones(K)
    prep = sq.prepare(W, s)
    Y = sq.linear(X, sq.inverse_scales_f32(s), prep)
    np.testing.assert_array_equal(Y, X @ W)
