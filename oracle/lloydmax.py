"""Lloyd-Max codebook activations with a closed-form per-token scale (oracle, test
infrastructure).

OrbitQuant (section 03): after the randomised permuted block-Hadamard rotation the
coordinates of a token are close to Gaussian whatever the input distribution, so one
Lloyd-Max codebook quantizes every layer and timestep without calibration data. CentriQ
(abstract): once each token is centred (the mean returns through the rank-1 branch), the
per-token scale follows in closed form without data.

Readings (the pages name the codebook and the closed form, nothing more):

* the codebook is the 16-level Lloyd-Max quantizer of the standard normal N(0, 1):
  thresholds are the midpoints of neighbouring levels and each level is the mean of
  N(0, 1) over its cell; the levels come from Lloyd's alternation of those two
  conditions, started from a uniform grid and run to a fixed point in float64;
* the per-token scale is sigma_m = sqrt(mean_k Xt[m, k]^2), the RMS of the rotated
  (centred) token: the rotated coordinates are then approximately N(0, sigma_m^2) and
  z = Xt / sigma_m meets the codebook's design distribution; for the orthonormal RPBH
  rotation sigma_m equals the RMS of the centred token before the rotation;
* a value takes the level nearest to z (its magnitude from the thresholds of |z|, a
  magnitude exactly on a threshold taking the larger level; the sign of z); a token with
  sigma_m = 0 is all zeros and stays zero;
* the tensor cores have no codebook format, so the decoded activation is handed to the
  contraction as an fp16 value fp16(fp32(sigma_m) * fp32(level)) (round to nearest
  even), and the weights' MXFP4 residual is decoded to fp16 the same way; the product is
  then an fp16 x fp16 contraction with fp32 accumulation.
"""
import numpy as np
from math import erf, erfc, exp, pi, sqrt

from . import mxfp4 as _mx
from . import transforms as _tr

LEVELS = 16


def _pdf(x: float) -> float:
    return exp(-0.5 * x * x) / sqrt(2.0 * pi)


def _cdf(x: float) -> float:
    return 0.5 * erfc(-x / sqrt(2.0)) if x < 0 else 0.5 * (1.0 + erf(x / sqrt(2.0)))


def gaussian_lloyd_max(n: int = LEVELS, tol: float = 1e-15, max_iter: int = 200000):
    """(levels [n] ascending, thresholds [n - 1]) of the n-level Lloyd-Max quantizer of
    N(0, 1), float64. Lloyd's alternation: thresholds <- midpoints of the levels;
    levels <- conditional means (pdf(a) - pdf(b)) / (cdf(b) - cdf(a)) over each cell,
    kept exactly symmetric about 0 (the density is)."""
    lv = np.linspace(-2.0, 2.0, n)
    for _ in range(max_iter):
        th = 0.5 * (lv[:-1] + lv[1:])
        edges = np.concatenate(([-np.inf], th, [np.inf]))
        new = np.empty(n)
        for i in range(n):
            a, b = edges[i], edges[i + 1]
            pa = 0.0 if np.isinf(a) else _pdf(a)
            pb = 0.0 if np.isinf(b) else _pdf(b)
            ca = 0.0 if np.isinf(a) else _cdf(a)
            cb = 1.0 if np.isinf(b) else _cdf(b)
            new[i] = (pa - pb) / (cb - ca)
        new = 0.5 * (new - new[::-1])    # N(0, 1) is symmetric: keep the levels exactly so
        done = np.max(np.abs(new - lv)) < tol
        lv = new
        if done:
            break
    return lv, 0.5 * (lv[:-1] + lv[1:])


def magnitudes(n: int = LEVELS):
    """(positive levels [n/2] ascending, their thresholds [n/2 - 1]) of the symmetric
    codebook; the decision between the two innermost levels -l1, +l1 is the sign."""
    lv, _ = gaussian_lloyd_max(n)
    pos = lv[n // 2:]
    return pos, 0.5 * (pos[:-1] + pos[1:])


def distortion(levels) -> float:
    """Mean squared error of the codebook on N(0, 1) (closed form per cell)."""
    lv = np.asarray(levels, dtype=np.float64)
    th = 0.5 * (lv[:-1] + lv[1:])
    edges = np.concatenate(([-np.inf], th, [np.inf]))
    d = 0.0
    for i, c in enumerate(lv):
        a, b = edges[i], edges[i + 1]
        pa = 0.0 if np.isinf(a) else _pdf(a)
        pb = 0.0 if np.isinf(b) else _pdf(b)
        ca = 0.0 if np.isinf(a) else _cdf(a)
        cb = 1.0 if np.isinf(b) else _cdf(b)
        ea = 0.0 if np.isinf(a) else a * pa
        eb = 0.0 if np.isinf(b) else b * pb
        m0 = cb - ca                     # P(cell)
        m1 = pa - pb                     # E[z; cell]
        m2 = m0 + ea - eb                # E[z^2; cell]
        d += m2 - 2.0 * c * m1 + c * c * m0
    return d


def token_sigma(Xt) -> np.ndarray:
    """sigma_m = sqrt(mean_k Xt[m, k]^2), float64 [M]."""
    Xt = np.asarray(Xt, dtype=np.float64)
    return np.sqrt(np.mean(Xt * Xt, axis=1))


def encode(Xt, sigma=None):
    """Codes uint8 [M, K] (sign << 3 | magnitude index 0..7) and sigma [M].
    z = Xt / sigma; the magnitude index counts the thresholds |z| reaches."""
    Xt = np.asarray(Xt, dtype=np.float64)
    sig = token_sigma(Xt) if sigma is None else np.asarray(sigma, dtype=np.float64)
    pos, th = magnitudes()
    with np.errstate(divide="ignore", invalid="ignore"):
        z = np.where(sig[:, None] > 0, Xt / sig[:, None], 0.0)
    idx = np.zeros(Xt.shape, dtype=np.int64)
    for t in th:
        idx += (np.abs(z) >= t)
    return ((np.signbit(z).astype(np.int64) << 3) | idx).astype(np.uint8), sig


def decode(codes, sigma) -> np.ndarray:
    """float64 sigma * level for codes from ``encode``."""
    pos, _ = magnitudes()
    c = np.asarray(codes).astype(np.int64)
    mag = pos[c & 7]
    return np.where(c & 8, -mag, mag) * np.asarray(sigma, dtype=np.float64)[:, None]


def fp16_operand(codes, sigma) -> np.ndarray:
    """The stored activation operand: fp16(fp32(sigma) * fp32(level)) with the code's
    sign, as float64."""
    pos, _ = magnitudes()
    c = np.asarray(codes).astype(np.int64)
    s32 = np.asarray(sigma, dtype=np.float64).astype(np.float32)
    mag = (s32[:, None] * pos.astype(np.float32)[c & 7]).astype(np.float16)
    return np.where(c & 8, -mag.astype(np.float64), mag.astype(np.float64))


def residual_fp16(prep: dict) -> np.ndarray:
    """The weights' MXFP4 residual decoded and rounded to fp16, [K, N] float64."""
    Rq = _mx.decode(prep["r_codes"], prep["r_scales"]).T
    return Rq.astype(np.float16).astype(np.float64)


def quantize_act(X, T: dict, centre_on: bool, prep: dict) -> dict:
    """The online half with the codebook in place of MXFP4 (centre, rotate, sigma, encode,
    fp16 operand; U on the unquantised rotated input as in the MXFP4 layer)."""
    X = np.asarray(X, dtype=np.float64)
    mu = X.mean(axis=1) if centre_on else np.zeros(X.shape[0])
    Xt = _tr.apply(X - mu[:, None], T)
    codes, sig = encode(Xt)
    return {"mu": mu, "Xt": Xt, "codes": codes, "sigma": sig,
            "A16": fp16_operand(codes, sig), "U": Xt @ prep["L1"]}


def linear(X, T: dict, centre_on: bool, prep: dict) -> np.ndarray:
    """Y = fp16 operand x fp16 residual + U L2 + mu s (float64)."""
    a = quantize_act(X, T, centre_on, prep)
    return a["A16"] @ residual_fp16(prep) + a["U"] @ prep["L2"] + np.outer(a["mu"], prep["s"])
