"""Robust l_p fit of MXFP4 block scales (oracle, test infrastructure).

CentriQ (summary and abstract) fits the weights "with a robust l_p objective that tracks
each group's dense mode while discounting heavy tails". The pages give neither p nor the
search; the reading taken here:

* a group is one MXFP4 block (32 consecutive elements along K of the residual R);
* candidates are the OCP exponent e0 = floor(log2 amax) - 2 and the n_down exponents
  below it (e0 - 1, ..., e0 - n_down, never below -127): a smaller scale saturates the
  block's largest values at +-6 * 2^e but resolves the bulk of the block more finely;
* for each candidate the codes are the usual ones (round to nearest, ties to even,
  saturate at +-6, sign bit kept), and the objective is sum_k |v_k - deq_k|^p in float64;
* the candidate with the smallest objective wins; ties go to the larger exponent (the
  OCP choice).

With n_down = 0 this is the plain OCP encoder.
"""
import numpy as np

from . import mxfp4 as _mx

BLOCK = _mx.BLOCK


def codes_at_exponent(v, e):
    """Codes of float32 values v (float64 array [..., 32]) at the forced exponent e
    (broadcast over the leading axes): RNE to the E2M1 grid of v / 2^e, saturating."""
    v = np.asarray(v, dtype=np.float64)
    w = v / np.exp2(np.asarray(e, dtype=np.float64))[..., None]
    mag = _mx._round_e2m1_magnitude(np.abs(w))
    return ((np.signbit(v).astype(np.int64) << 3) | mag).astype(np.uint8)


def lp_error(v, codes, e, p: float):
    """sum_k |v_k - e2m1(code_k) 2^e|^p over the last axis (float64)."""
    deq = _mx.e2m1_value(codes) * np.exp2(np.asarray(e, dtype=np.float64))[..., None]
    return np.sum(np.abs(np.asarray(v, dtype=np.float64) - deq) ** p, axis=-1)


def encode_lp(v, p: float, n_down: int = 3):
    """(codes uint8 [..., K], scales uint8 [..., K/32], objective [..., K/32]).

    v: float32 values given as float64, K % 32 == 0."""
    v = np.asarray(v, dtype=np.float64)
    if v.shape[-1] % BLOCK:
        raise ValueError("K must be a multiple of 32")
    if np.any(v.astype(np.float32).astype(np.float64) != v):
        raise ValueError("encoder input must be exactly float32")
    blk = v.reshape(v.shape[:-1] + (v.shape[-1] // BLOCK, BLOCK))
    e0 = _mx.shared_exponent(np.max(np.abs(blk), axis=-1))
    best_e = e0.copy()
    best_c = codes_at_exponent(blk, e0)
    best_f = lp_error(blk, best_c, e0, p)
    for d in range(1, n_down + 1):
        e = np.maximum(e0 - d, -127)
        c = codes_at_exponent(blk, e)
        f = lp_error(blk, c, e, p)
        better = f < best_f                        # strict: ties keep the larger exponent
        best_e = np.where(better, e, best_e)
        best_c = np.where(better[..., None], c, best_c)
        best_f = np.where(better, f, best_f)
    return (best_c.reshape(v.shape), (best_e + _mx.SCALE_BIAS).astype(np.uint8),
            best_f)


def objective_gap(v, p: float, n_down: int = 3):
    """Relative gap between the best and the second-best candidate objective per block
    (tests accept a different choice only where this gap is below rounding level)."""
    v = np.asarray(v, dtype=np.float64)
    blk = v.reshape(v.shape[:-1] + (v.shape[-1] // BLOCK, BLOCK))
    e0 = _mx.shared_exponent(np.max(np.abs(blk), axis=-1))
    fs = []
    for d in range(0, n_down + 1):
        e = np.maximum(e0 - d, -127)
        fs.append(lp_error(blk, codes_at_exponent(blk, e), e, p))
    f = np.sort(np.stack(fs, axis=-1), axis=-1)
    return (f[..., 1] - f[..., 0]) / np.maximum(f[..., 1], 1e-300)
