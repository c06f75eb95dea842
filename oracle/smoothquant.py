"""SmoothQuant-style per-channel scaling followed by MXFP4 (oracle, test infrastructure).

The comparator the KroQuant commentary measures its quantization kernel against
(section 02: on MI350 the KroQuant kernel is up to 14 % faster than SmoothQuant's
channel-wise scaling; section 01: channel-wise scaling is cheap but too weak for W4A4).
SmoothQuant migrates activation outliers into the weight with one scale per input
channel: X W = (X diag(s)^-1)(diag(s) W).

Scale rule (SmoothQuant's migration strength alpha; the commentary does not restate it,
so the original rule is used): s_j = max_m |X[m, j]|^alpha / max_n |W[j, n]|^(1 - alpha),
computed in float64 from calibration statistics; channels whose maxima are zero get
s_j = 1.

Online half: the activation is multiplied by the float32 reciprocal inv_s = fp32(1/s)
and the product, rounded to float32, is MXFP4-encoded along K. (The kernel takes the
same float32 multiply, so the code decisions are made in the same precision.)
Offline half: W_s = diag(s) W, rounded to float32 and MXFP4-encoded along K.
Output: Y = deq(Q(X * inv_s)) deq(Q(W_s)).
"""
import numpy as np

from . import mxfp4 as _mx


def smooth_scales(x_absmax, w_absmax, alpha: float = 0.5) -> np.ndarray:
    """Per-channel SmoothQuant scales s [K] (float64) from channel maxima of X and W."""
    xa = np.asarray(x_absmax, dtype=np.float64)
    wa = np.asarray(w_absmax, dtype=np.float64)
    s = np.ones_like(xa)
    ok = (xa > 0) & (wa > 0)
    s[ok] = xa[ok] ** alpha / wa[ok] ** (1.0 - alpha)
    return s


def scales_from(X, W, alpha: float = 0.5) -> np.ndarray:
    """s from the activation batch itself (stands in for calibration data) and W [K, N]."""
    X = np.asarray(X, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    return smooth_scales(np.abs(X).max(axis=0), np.abs(W).max(axis=1), alpha)


def inverse_scales_f32(s) -> np.ndarray:
    """The float32 reciprocals the online half multiplies by."""
    return (1.0 / np.asarray(s, dtype=np.float64)).astype(np.float32)


def scale_act(X, inv_s32) -> np.ndarray:
    """X * inv_s per channel, each product rounded to float32 (returned as float64)."""
    Xf = np.asarray(X, dtype=np.float32)               # bf16 values are exact in fp32
    return (Xf * np.asarray(inv_s32, dtype=np.float32)[None, :]).astype(np.float64)


def quantize_act(X, inv_s32) -> dict:
    """Codes [M, K] (one per element) and E8M0 scales [M, K/32] of the scaled activation."""
    Xs = scale_act(X, inv_s32)
    codes, scales = _mx.encode(Xs)
    return {"Xs": Xs, "codes": codes, "scales": scales}


def smooth_weight(W, s) -> np.ndarray:
    """diag(s) W in float64."""
    return np.asarray(s, dtype=np.float64)[:, None] * np.asarray(W, dtype=np.float64)


def prepare(W, s) -> dict:
    """W_s = diag(s) W rounded to float32 and MXFP4-encoded along K (per output column)."""
    Ws = smooth_weight(W, s)
    Ws32 = Ws.astype(np.float32).astype(np.float64)
    codes_t, scales_t = _mx.encode(Ws32.T)               # [N, K] rows: blocks along K
    return {"Ws": Ws, "Ws32": Ws32, "r_codes": codes_t, "r_scales": scales_t}


def linear(X, inv_s32, prep: dict) -> np.ndarray:
    """Y = deq(Q(X * inv_s)) deq(Q(W_s)) in float64."""
    act = quantize_act(X, inv_s32)
    Xd = _mx.decode(act["codes"], act["scales"])
    Wd = _mx.decode(prep["r_codes"], prep["r_scales"])
    return Xd @ Wd.T
