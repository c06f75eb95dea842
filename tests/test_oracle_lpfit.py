"""Pins of the robust l_p scale fit: brute force over forced exponents and codes,
reduction to the OCP encoder, exact power-of-two invariance, and hand-derived blocks
where the choice of p decides between tracking the bulk and keeping the outlier."""
import numpy as np
import pytest

from oracle import lpfit, mxfp4


def _v(seed, rows=6, K=96, tail=True):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((rows, K))
    if tail:
        v[rng.random((rows, K)) < 0.04] *= 25.0         # heavy-tailed groups
    return v.astype(np.float32).astype(np.float64)


def _brute(v, p, n_down):
    """Independent search: for every candidate exponent, every element takes the code
    (among the 8 magnitudes with the element's sign) nearest to v/2^e, ties to the code
    with an even index; the block objective is summed and minimised, ties to larger e."""
    mags = mxfp4.e2m1_value(np.arange(8))
    codes = np.zeros(v.shape, np.uint8)
    scales = np.zeros(v.shape[:-1] + (v.shape[-1] // 32,), np.uint8)
    for idx in np.ndindex(*v.shape[:-1]):
        for b in range(v.shape[-1] // 32):
            x = v[idx][32 * b:32 * b + 32]
            amax = np.abs(x).max()
            e0 = -127 if amax == 0 else int(np.clip(np.floor(np.log2(amax)) - 2, -127, 127))
            best = None
            for d in range(n_down + 1):
                e = max(e0 - d, -127)
                cs, f = [], 0.0
                for xi in x:
                    w = abs(xi) / 2.0 ** e
                    dist = np.abs(mags - w)
                    m = int(np.argmin(dist))                  # first minimum = lower index
                    if m + 1 < 8 and dist[m + 1] == dist[m] and m % 2 == 1:
                        m += 1
                    cs.append((8 if np.signbit(xi) else 0) | m)
                    f += abs(xi - np.sign(xi) * mags[m] * 2.0 ** e) ** p
                if best is None or f < best[0]:
                    best = (f, e, cs)
            codes[idx + (slice(32 * b, 32 * b + 32),)] = best[2]
            scales[idx + (b,)] = best[1] + 127
    return codes, scales


@pytest.mark.parametrize("p", [0.5, 1.0, 2.0])
def test_matches_bruteforce(p):
    v = _v(1, rows=3, K=64)
    c, s, _ = lpfit.encode_lp(v, p)
    cb, sb = _brute(v, p, 3)
    np.testing.assert_array_equal(s, sb)
    np.testing.assert_array_equal(c, cb)


def test_no_search_is_the_ocp_encoder():
    v = _v(2)
    c, s, _ = lpfit.encode_lp(v, 1.0, n_down=0)
    c0, s0 = mxfp4.encode(v)
    np.testing.assert_array_equal(c, c0)
    np.testing.assert_array_equal(s, s0)


@pytest.mark.parametrize("k", [-7, 4])
def test_power_of_two_invariance(k):
    v = _v(3)
    c, s, f = lpfit.encode_lp(v, 1.0)
    c2, s2, f2 = lpfit.encode_lp(v * 2.0 ** k, 1.0)
    np.testing.assert_array_equal(c2, c)
    np.testing.assert_array_equal(s2.astype(int), s.astype(int) + k)
    np.testing.assert_allclose(f2, f * 2.0 ** k, rtol=1e-15)


def test_objective_never_worse_than_ocp():
    v = _v(4, rows=20)
    for p in (0.5, 1.0, 2.0):
        c, s, f = lpfit.encode_lp(v, p)
        c0, s0 = mxfp4.encode(v)
        blk = v.reshape(v.shape[0], -1, 32)
        f0 = lpfit.lp_error(blk, c0.reshape(blk.shape), s0.astype(np.int64) - 127, p)
        assert np.all(f <= f0)


def test_outlier_block_p_decides():
    """31 values 0.75 and one 100 (worked by hand). OCP: e0 = 4, the bulk rounds to 0
    (|err| 0.75 each) and 100 -> 96: l1 = 27.25, l0.5 = 31 sqrt(.75) + 2 = 28.85.
    e0 - 3 = 1: the bulk becomes 1.0 (|err| .25 each), 100 saturates at 12:
    l1 = 7.75 + 88 = 95.75, l0.5 = 15.5 + sqrt(88) = 24.88.
    e0 - 1 = 3: bulk 0.75/8 -> 0 (0.09375 < .25), 100/8 = 12.5 -> 6: 48, l1 = 23.25 + 52 = 75.25;
    e0 - 2 = 2: bulk 0.75/4 = .1875 -> 0, 100/4 = 25 -> 6: 24: l1 = 23.25 + 76 = 99.25,
    l0.5 = 26.85 + 8.72 = 35.6; e0 - 1 l0.5 = 26.85 + 7.21 = 34.06.
    So l1 keeps the OCP scale and l0.5 tracks the bulk (e0 - 3)."""
    v = np.full((1, 32), 0.75)
    v[0, 5] = 100.0
    c1, s1, f1 = lpfit.encode_lp(v, 1.0)
    assert int(s1[0, 0]) - 127 == 4
    np.testing.assert_allclose(f1[0, 0], 27.25)
    ch, sh, fh = lpfit.encode_lp(v, 0.5)
    assert int(sh[0, 0]) - 127 == 1
    np.testing.assert_allclose(fh[0, 0], 15.5 + np.sqrt(88.0))
    assert mxfp4.e2m1_value(ch[0, 0]) == 0.5 and mxfp4.e2m1_value(ch[0, 5]) == 6.0


def test_exact_block_keeps_ocp_scale():
    """32 copies of 1.5 * 2^k are exact at e0 (value 6); every smaller scale saturates."""
    for k in (-3, 0, 5):
        v = np.full((1, 32), 1.5 * 2.0 ** k)
        c, s, f = lpfit.encode_lp(v, 1.0)
        assert int(s[0, 0]) - 127 == k - 2 and f[0, 0] == 0.0
