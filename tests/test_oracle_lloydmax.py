"""Pins of the Lloyd-Max codebook oracle: the published 16-level Gaussian table, the
two-level closed form, the optimality conditions and the distortion by independent
numerical quadrature, a brute-force nearest-level encoder, the scale invariance of the
per-token sigma under the orthonormal rotation, and the fp16 operand rounding."""
import os

import numpy as np
import pytest
from scipy import integrate, stats

from oracle import lloydmax as lm
from oracle import transforms
from synthetic import make_inputs, workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "lloydmax_gaussian16.txt")


def _max_table():
    """Max (1960), Table I, N = 16 (tests/golden/lloydmax_gaussian16.txt): the positive
    decision levels and output levels, 4 decimals."""
    rows = [ln.split() for ln in open(GOLDEN) if ln.strip() and not ln.startswith("#")]
    x = np.array([float(r[0]) for r in rows])
    y = np.array([float(r[1]) for r in rows])
    return x, y


def test_matches_published_table():
    lv, th = lm.gaussian_lloyd_max(16)
    x, y = _max_table()
    np.testing.assert_allclose(lv[8:], y, atol=6e-4)
    np.testing.assert_allclose(th[7:], x, atol=6e-4)            # th[7] = 0: the sign decision
    np.testing.assert_array_equal(lv[:8], -lv[8:][::-1])                # symmetric


def test_two_levels_closed_form():
    """Two levels: +-E[|z|] = +-sqrt(2/pi), distortion 1 - 2/pi."""
    lv, th = lm.gaussian_lloyd_max(2)
    np.testing.assert_allclose(lv, [-np.sqrt(2 / np.pi), np.sqrt(2 / np.pi)], rtol=1e-12)
    np.testing.assert_allclose(lm.distortion(lv), 1 - 2 / np.pi, rtol=1e-12)


def test_optimality_by_quadrature():
    """Every level is the mean of N(0,1) over its cell and the distortion equals the
    integral of (z - level)^2, both by adaptive quadrature (independent of the oracle's
    closed forms)."""
    lv, th = lm.gaussian_lloyd_max(16)
    np.testing.assert_allclose(th, 0.5 * (lv[:-1] + lv[1:]), rtol=0, atol=0)
    edges = np.concatenate(([-np.inf], th, [np.inf]))
    phi = stats.norm.pdf
    D = 0.0
    for i, c in enumerate(lv):
        a, b = edges[i], edges[i + 1]
        p = integrate.quad(phi, a, b, epsabs=1e-14, epsrel=1e-13)[0]
        m = integrate.quad(lambda z: z * phi(z), a, b, epsabs=1e-14, epsrel=1e-13)[0]
        D += integrate.quad(lambda z: (z - c) ** 2 * phi(z), a, b, epsabs=1e-14, epsrel=1e-13)[0]
        assert abs(m / p - c) < 1e-11
    np.testing.assert_allclose(lm.distortion(lv), D, rtol=1e-10)
    assert 0.00949 < D < 0.00951


def test_local_optimality():
    """Moving any one level away from the fixed point raises the distortion."""
    lv, _ = lm.gaussian_lloyd_max(16)
    d0 = lm.distortion(lv)
    for i in range(16):
        for eps in (1e-3, -1e-3):
            v = lv.copy()
            v[i] += eps
            assert lm.distortion(np.sort(v)) > d0


def test_encoder_is_nearest_level():
    rng = np.random.default_rng(5)
    Xt = rng.standard_normal((40, 256)) * rng.uniform(0.1, 30, (40, 1))
    Xt[rng.random(Xt.shape) < 0.01] *= 20
    codes, sig = lm.encode(Xt)
    lv, _ = lm.gaussian_lloyd_max(16)
    z = Xt / sig[:, None]
    nearest = lv[np.argmin(np.abs(z[..., None] - lv), axis=-1)]
    np.testing.assert_array_equal(lm.decode(codes, np.ones(40)), nearest)
    # decoding and encoding again at the same sigma gives the same codes
    again, _ = lm.encode(lm.decode(codes, sig), sig)
    np.testing.assert_array_equal(again, codes)


def test_empirical_distortion_on_gaussian_data():
    rng = np.random.default_rng(6)
    z = rng.standard_normal((64, 4096))
    codes, sig = lm.encode(z, np.ones(64))
    mse = np.mean((lm.decode(codes, np.ones(64)) - z) ** 2)
    assert abs(mse / lm.distortion(lm.gaussian_lloyd_max(16)[0]) - 1) < 0.03


def test_sigma_is_rotation_invariant():
    """RPBH is orthonormal: the RMS of the rotated, centred token equals the RMS of the
    centred token (the kernel forms sigma before the rotation)."""
    w = workload(2, M=16, K=256, N=64)
    inp = make_inputs(w)
    X = inp["X"].double().numpy()
    Xc = X - X.mean(axis=1, keepdims=True)
    Xt = transforms.apply(Xc, inp["T"])
    np.testing.assert_allclose(lm.token_sigma(Xt), np.sqrt(np.mean(Xc ** 2, axis=1)), rtol=1e-13)


def test_zero_token_and_fp16_operand():
    Xt = np.zeros((2, 64))
    Xt[1] = np.linspace(-3, 3, 64)
    codes, sig = lm.encode(Xt)
    assert sig[0] == 0 and np.all(lm.decode(codes, sig)[0] == 0)
    A = lm.fp16_operand(codes, sig)
    assert np.all(A[0] == 0)
    d = lm.decode(codes, sig)
    assert np.all(np.abs(A - d) <= 2.0 ** -11 * np.abs(d) + 1e-30)
    assert np.all(A.astype(np.float16).astype(np.float64) == A)        # exact fp16 values
