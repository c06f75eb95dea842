"""MXFP4 encode/decode (oracle, test infrastructure).

The KroQuant commentary (section 03) quantizes to MXFP4; the format is defined
by the OCP Microscaling Formats (MX) v1.0 specification:

* elements are FP4 E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit;
  magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}; code = sign<<3 | exponent<<1 | mantissa;
* one E8M0 shared scale per block of 32 consecutive elements along K:
  a pure power of two 2^e stored as the byte e + 127;
* the shared exponent is floor(log2(amax)) - emax_elem with emax_elem = 2
  (the largest E2M1 power of two, 4 = 2^2), clamped to the E8M0 range
  [-127, 127];
* each element is v / 2^e rounded to nearest, ties to even mantissa, and
  saturated to +-6.

Readings taken where the pages say nothing beyond the name "MXFP4":
* the encoder input is a float32 value (given here as exact float64);
* floor(log2(amax)) is taken exactly (``frexp``), never from a floating log;
* the code's sign bit is the input's sign bit, so a negative value that
  rounds to zero gives code 0x8 (-0), and -0.0 gives 0x8;
* an all-zero block gets the smallest scale, byte 0x00 (e = -127).

``encode`` is the closed form; ``encode_bruteforce`` (used by the pins) is
the definition "nearest of the 16 codes, ties to even mantissa" searched
exhaustively.
"""
import numpy as np

# magnitudes of the 8 non-negative E2M1 codes 0..7 (exponent bias 1):
# code 0: 0, code 1: subnormal 0.5, codes 2..7: 2^(E-1) * (1 + M/2)
E2M1_MAGNITUDE = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
BLOCK = 32
EMAX_ELEM = 2
SCALE_BIAS = 127


def e2m1_value(code) -> np.ndarray:
    """float64 value of 4-bit codes 0..15."""
    code = np.asarray(code).astype(np.int64)
    mag = E2M1_MAGNITUDE[code & 7]
    return np.where(code & 8, -mag, mag)


def shared_exponent(amax) -> np.ndarray:
    """e = clamp(floor(log2(amax)) - 2, -127, 127); amax == 0 gives -127."""
    amax = np.asarray(amax, dtype=np.float64)
    _, ex = np.frexp(amax)          # amax = m * 2**ex, 0.5 <= m < 1  ->  floor(log2) = ex - 1
    e = (ex - 1) - EMAX_ELEM
    e = np.where(amax == 0, -SCALE_BIAS, e)
    return np.clip(e, -SCALE_BIAS, SCALE_BIAS).astype(np.int64)


def _round_e2m1_magnitude(a) -> np.ndarray:
    """Closed-form round-to-nearest-even of magnitudes a >= 0 onto the E2M1 grid,
    saturating at 6. Returns the 3-bit magnitude code 0..7.

    Decision points are the midpoints between neighbouring grid values; at an
    exact midpoint the code with mantissa bit 0 (an even code) wins."""
    a = np.asarray(a, dtype=np.float64)
    mids = (E2M1_MAGNITUDE[1:] + E2M1_MAGNITUDE[:-1]) / 2.0     # 0.25 .75 1.25 1.75 2.5 3.5 5
    code = np.searchsorted(mids, a, side="left")               # count of midpoints < a
    at_mid = np.isin(a, mids)
    # at a midpoint, searchsorted(side=left) returns the lower neighbour i; pick the even one
    code = np.where(at_mid & (code % 2 == 1), code + 1, code)
    return np.minimum(code, 7).astype(np.int64)


def encode(v):
    """Encode rows of float32 values (given as float64) blockwise along the last axis.

    v: [..., K] with K % 32 == 0.  Returns (codes uint8 [..., K] in 0..15,
    scales uint8 [..., K/32] = e + 127)."""
    v = np.asarray(v, dtype=np.float64)
    if v.shape[-1] % BLOCK:
        raise ValueError("K must be a multiple of 32")
    if not np.all(np.isfinite(v)):
        raise ValueError("non-finite encoder input is outside the contract")
    if np.any(v.astype(np.float32).astype(np.float64) != v):
        raise ValueError("encoder input must be exactly float32")
    blk = v.reshape(v.shape[:-1] + (v.shape[-1] // BLOCK, BLOCK))
    amax = np.max(np.abs(blk), axis=-1)
    e = shared_exponent(amax)
    w = blk / np.exp2(e.astype(np.float64))[..., None]          # exact power-of-two scaling
    mag = _round_e2m1_magnitude(np.abs(w))
    sign = np.signbit(blk).astype(np.int64)
    codes = (sign << 3) | mag
    return codes.reshape(v.shape).astype(np.uint8), (e + SCALE_BIAS).astype(np.uint8)


def encode_bruteforce(v):
    """Same contract as ``encode``, by exhaustive search over the 16 codes per
    element: minimise |v / 2^e - value(code)| among codes whose sign bit equals
    the input's sign bit; ties go to the code with mantissa bit 0.
    Saturation follows because |value| <= 6 for every code."""
    v = np.asarray(v, dtype=np.float64)
    blk = v.reshape(v.shape[:-1] + (v.shape[-1] // BLOCK, BLOCK))
    amax = np.max(np.abs(blk), axis=-1)
    # floor(log2(amax)) by a plain search over integers (independent of frexp)
    flo = np.full(amax.shape, -1000, dtype=np.int64)
    for k in range(-160, 130):
        flo = np.where((amax > 0) & (amax >= 2.0 ** k), k, flo)
    e = np.clip(np.where(amax == 0, -127, flo - 2), -127, 127)
    w = blk / (2.0 ** e.astype(np.float64))[..., None]
    neg = np.signbit(blk)
    best = np.zeros(blk.shape, dtype=np.int64)
    best_d = np.full(blk.shape, np.inf)
    for c in range(16):
        val = e2m1_value(c)
        ok = neg == bool(c & 8)
        d = np.abs(w - val)
        better = ok & ((d < best_d) | ((d == best_d) & (c % 2 == 0) & (best % 2 == 1)))
        best = np.where(better, c, best)
        best_d = np.where(better, d, best_d)
    return best.reshape(v.shape).astype(np.uint8), (e + 127).astype(np.uint8)


def decode(codes, scales) -> np.ndarray:
    """float64 values e2m1(code) * 2^(scale - 127), blockwise along the last axis."""
    codes = np.asarray(codes)
    scales = np.asarray(scales).astype(np.int64)
    vals = e2m1_value(codes)
    blk = vals.reshape(vals.shape[:-1] + (vals.shape[-1] // BLOCK, BLOCK))
    return (blk * np.exp2((scales - SCALE_BIAS).astype(np.float64))[..., None]).reshape(vals.shape)


def decision_margin(v) -> np.ndarray:
    """Distance of each element to its nearest rounding decision point, in units of its
    block's maximum magnitude: min_i | |v| - mid_i * 2^e | / amax, where mid_i are the
    midpoints between E2M1 grid values; and, for the whole block, the relative distance
    of amax to the nearest power of two (where the shared scale changes).

    Used by tests to accept code differences caused only by a last-ulp difference of a
    float32 value computed in another order. The unit is the block maximum because that
    is the unit in which a transform's rounding error is bounded (a Hadamard output can be
    much smaller than its inputs)."""
    v = np.asarray(v, dtype=np.float64)
    blk = v.reshape(v.shape[:-1] + (v.shape[-1] // BLOCK, BLOCK))
    amax = np.max(np.abs(blk), axis=-1, keepdims=True)
    e = shared_exponent(amax[..., 0])[..., None]
    scale = np.exp2(e.astype(np.float64))
    w = np.abs(blk) / scale
    mids = (E2M1_MAGNITUDE[1:] + E2M1_MAGNITUDE[:-1]) / 2.0
    d = np.min(np.abs(w[..., None] - mids), axis=-1) * scale / np.maximum(amax, 1e-300)
    la = np.log2(np.maximum(amax, 1e-300))
    dscale = np.abs(la - np.rint(la)) * np.log(2.0)
    d = np.minimum(d, np.broadcast_to(dscale, d.shape))
    return d.reshape(v.shape)
