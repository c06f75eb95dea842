"""Pins for the oracle's MXFP4 encoder/decoder (CPU only).

The closed-form encoder is checked against (a) an exhaustive nearest-code search,
(b) hand-derived blocks in tests/golden/mxfp4_blocks.txt, (c) the E2M1 value
formula of the OCP MX v1.0 specification written out independently here, and
(d) round-trip properties."""
import os

import numpy as np
import pytest

from oracle import mxfp4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mxfp4_blocks.txt")


def load_golden():
    cases, cur = [], None
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, _, rest = line.partition(" ")
        if key == "case":
            cur = {"name": rest.strip()}
            cases.append(cur)
        elif key == "values":
            v = np.zeros(32)
            vals = [float(t) for t in rest.split()]
            v[:len(vals)] = vals
            cur["values"] = v.astype(np.float32).astype(np.float64)
        elif key == "scale":
            cur["scale"] = int(rest)
        elif key == "codes":
            c = np.zeros(32, dtype=np.uint8)
            cs = [int(t, 16) for t in rest.split()]
            c[:len(cs)] = cs
            cur["codes"] = c
    return cases


@pytest.mark.parametrize("case", load_golden(), ids=lambda c: c["name"])
def test_hand_derived_blocks(case):
    codes, scales = mxfp4.encode(case["values"][None, :])
    assert int(scales[0, 0]) == case["scale"]
    np.testing.assert_array_equal(codes[0], case["codes"])
    bc, bs = mxfp4.encode_bruteforce(case["values"][None, :])
    np.testing.assert_array_equal(bc[0], case["codes"])
    assert int(bs[0, 0]) == case["scale"]


def test_e2m1_value_formula():
    # OCP MX v1.0 E2M1: sign s, exponent E (2 bits, bias 1), mantissa M (1 bit);
    # E == 0: (-1)^s * 2^(1-1) * (0 + M/2); E > 0: (-1)^s * 2^(E-1) * (1 + M/2)
    for c in range(16):
        s, E, M = c >> 3, (c >> 1) & 3, c & 1
        want = (0.5 * M) if E == 0 else (2.0 ** (E - 1)) * (1.0 + M / 2.0)
        want = -want if s else want
        assert mxfp4.e2m1_value(c) == want


def _random_blocks(rng, rows, scale_exp_range=(-20, 20)):
    v = rng.standard_normal((rows, 32)) * np.exp2(rng.integers(*scale_exp_range, size=(rows, 1)))
    heavy = rng.standard_t(2, size=(rows, 32)) * 3
    v = np.where(rng.random((rows, 32)) < 0.1, heavy, v)
    return v.astype(np.float32).astype(np.float64)


def test_closed_form_equals_bruteforce_random():
    rng = np.random.default_rng(123)
    v = _random_blocks(rng, 4000).reshape(-1, 32 * 4)
    c1, s1 = mxfp4.encode(v)
    c2, s2 = mxfp4.encode_bruteforce(v)
    np.testing.assert_array_equal(s1, s2)
    np.testing.assert_array_equal(c1, c2)


def test_closed_form_equals_bruteforce_adversarial():
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    mids = (grid[1:] + grid[:-1]) / 2
    rows = []
    for e in (-127, -126, -20, -3, 0, 5, 100, 124):
        base = np.concatenate([mids, -mids, grid, -grid, [6.0 + 0.5, 7.99, -7.99, 5.99],
                               [0.0, -0.0]])[:32]
        for amax_val in (6.0, 4.0, 7.5, 4.0 * (1 - 2 ** -23)):
            b = base.copy()
            b[0] = amax_val
            b = np.clip(b, -amax_val, amax_val)
            rows.append(b * 2.0 ** e)
    # exact powers of two as the block maximum, and values just below / above them
    for k in range(-130, 127, 7):
        p = 2.0 ** k
        rows.append(np.array([p, p * (1 - 2 ** -24), p / 2, p / 4, p / 8, p * 0.75,
                              p * 0.375, p * 0.1875] + [0.0] * 24))
    v = np.array(rows).astype(np.float32).astype(np.float64)
    c1, s1 = mxfp4.encode(v)
    c2, s2 = mxfp4.encode_bruteforce(v)
    np.testing.assert_array_equal(s1, s2)
    np.testing.assert_array_equal(c1, c2)


def test_exhaustive_bf16_patterns():
    """Every finite bf16 bit pattern as a block value, in two block settings:
    alone (it is the block maximum) and beside a fixed anchor of magnitude 1."""
    bits = np.arange(65536, dtype=np.uint32)
    vals = (bits << 16).view(np.float32).astype(np.float64)
    vals = vals[np.isfinite(vals)]
    pad = (-len(vals)) % 31
    vals = np.concatenate([vals, np.zeros(pad)])
    alone = np.zeros((len(vals), 32))
    alone[:, 0] = vals
    anchored = np.zeros((len(vals), 32))
    anchored[:, 0] = vals
    anchored[:, 1] = 1.0
    anchored[:, 2] = -0.75
    for v in (alone, anchored):
        c1, s1 = mxfp4.encode(v)
        c2, s2 = mxfp4.encode_bruteforce(v)
        np.testing.assert_array_equal(s1, s2)
        np.testing.assert_array_equal(c1, c2)


def test_roundtrip_and_error_bound():
    rng = np.random.default_rng(7)
    v = _random_blocks(rng, 2000).reshape(-1, 64)
    codes, scales = mxfp4.encode(v)
    d = mxfp4.decode(codes, scales)
    blk = v.reshape(-1, 32)
    e = scales.reshape(-1).astype(np.int64) - 127
    err = np.abs(d.reshape(-1, 32) - blk)
    # inside the grid the error is at most half a grid step: 0.25 below 2, 0.5 up to 4,
    # 1 up to 6 (times 2^e); values clipped at 6 lose at most amax - 6*2^e < 2*2^e
    bound = np.where(np.abs(blk) / np.exp2(e)[:, None] > 6, 2.0, 1.0) * np.exp2(e)[:, None]
    assert np.all(err <= bound + 0)
    # decoded values are exactly representable and re-encode to the same codes
    c2, s2 = mxfp4.encode(d)
    np.testing.assert_array_equal(s2, scales)
    np.testing.assert_array_equal(c2 & 7, codes & 7)


def test_scale_is_largest_exponent_not_clipping_beyond_8():
    # the scale rule guarantees amax / 2^e in [4, 8): the maximum never needs more than 2x clip
    rng = np.random.default_rng(3)
    v = _random_blocks(rng, 3000)
    _, s = mxfp4.encode(v)
    amax = np.abs(v).max(axis=1)
    r = amax / np.exp2(s[:, 0].astype(np.int64) - 127)
    ok = amax > 2.0 ** -120
    assert np.all((r[ok] >= 4) & (r[ok] < 8))


def test_input_contract():
    with pytest.raises(ValueError):
        mxfp4.encode(np.full((1, 32), 0.1))          # not a float32 value
    with pytest.raises(ValueError):
        mxfp4.encode(np.full((1, 31), 1.0))          # K not a multiple of 32
    with pytest.raises(ValueError):
        mxfp4.encode(np.array([[np.inf] + [0.0] * 31]))
