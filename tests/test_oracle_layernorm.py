"""Pins of the LayerNorm front-end oracle: a hand-computed row, the defining moments,
invariance to a per-token shift, the affine, and the algebraic decomposition the GPU's
low-rank kernel uses to form y L1' from raw activations."""
import os

import numpy as np

from oracle import layernorm as ln

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "layernorm_rows.txt")


def _golden():
    cases, cur = [], None
    for line in open(GOLDEN):
        t = line.split()
        if not t or t[0].startswith("#"):
            continue
        if t[0] == "case":
            cur = {"name": t[1]}
            cases.append(cur)
        else:
            cur[t[0]] = np.array([float(v) for v in t[1:]])
    return cases


def test_golden_rows():
    cases = _golden()
    assert len(cases) == 3
    for c in cases:
        y = ln.layernorm(c["x"][None, :], c["gamma"], c["beta"], float(c["eps"][0]))
        np.testing.assert_allclose(y[0], c["y"], rtol=1e-15, atol=1e-15, err_msg=c["name"])


def test_hand_row():
    """x = (1, 2, 3, 4): m = 2.5, v = 1.25, y = (x - 2.5) / sqrt(1.25)."""
    y = ln.layernorm(np.array([[1.0, 2.0, 3.0, 4.0]]), np.ones(4), np.zeros(4), 0.0)
    r = 1.0 / np.sqrt(1.25)
    np.testing.assert_allclose(y, [[-1.5 * r, -0.5 * r, 0.5 * r, 1.5 * r]], rtol=1e-15)


def test_moments_without_affine():
    rng = np.random.default_rng(0)
    X = rng.standard_normal((16, 96)) * rng.uniform(0.1, 9, (16, 1)) + rng.normal(0, 5, (16, 1))
    eps = 1e-6
    y = ln.layernorm(X, np.ones(96), np.zeros(96), eps)
    np.testing.assert_allclose(y.mean(axis=1), 0.0, atol=1e-13)
    v = X.var(axis=1)
    np.testing.assert_allclose(y.var(axis=1), v / (v + eps), rtol=1e-12)


def test_shift_invariance_and_affine():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((8, 64))
    g = rng.uniform(0.5, 2, 64)
    b = rng.normal(0, 1, 64)
    y0 = ln.layernorm(X, g, b, 1e-5)
    y1 = ln.layernorm(X + rng.normal(0, 30, (8, 1)), g, b, 1e-5)
    np.testing.assert_allclose(y1, y0, rtol=1e-9, atol=1e-9)
    plain = ln.layernorm(X, np.ones(64), np.zeros(64), 1e-5)
    np.testing.assert_allclose(y0, plain * g + b, rtol=1e-14, atol=1e-14)


def test_lowrank_decomposition():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((10, 64)) * 3 + rng.normal(0, 4, (10, 1))
    g = rng.uniform(0.5, 2, 64)
    b = rng.normal(0, 1, 64)
    L1p = rng.standard_normal((64, 7))
    direct, decomposed = ln.lowrank_input_parts(X, g, b, 1e-6, L1p)
    np.testing.assert_allclose(decomposed, direct, rtol=1e-10, atol=1e-10)
