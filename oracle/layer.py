"""The W4A4 quantized linear layer, step by step (oracle, test infrastructure).

Row-vector convention: Y = X W with X [M, K] (tokens x features), W [K, N].

Online half, per token (``quantize_act``):
 1. centring (CentriQ abstract: centre each token before the rotation):
    mu_m = mean_k X[m, k], X_c = X - mu 1^T.  Off when the layer does not centre.
 2. block transform Xt = X_c P (KroQuant section 02 / OrbitQuant section 03),
    see ``oracle.transforms``.
 3. MXFP4 encode of Xt along K (KroQuant section 03 names MXFP4), after
    rounding Xt to float32, the encoder's input type.
 4. low-rank input U = Xt L1, kept unrounded here (SVDQuant explainer,
    section 3: the low-rank branch runs in 16-bit on the unquantised input).

Offline half, per layer (``prepare``; OrbitQuant section 03: the inverse is
absorbed into the next weight once, offline):
 5. s = 1^T W, column sums of the ORIGINAL weight (CentriQ: the rank-1
    full-precision branch restores the mean exactly because X W = X_c W + mu s).
 6. W' = P^{-1} W (KroQuant section 01: Y = (X P)(P^{-1} W)).
 7. truncated SVD of W' (SVDQuant section 3: SVD of the updated weight, the top
    r singular components kept at 16-bit): W' = U S V^T, L1 = bf16(U_r sqrt(S_r)),
    L2 = bf16(sqrt(S_r) V_r^T).
 8. residual R = W' - L1 L2 with the rounded factors, rounded to float32 and
    MXFP4-encoded along K (SVDQuant section 3: the residual goes to 4 bits).
 9. L1' = P L1 and c1 = 1^T L1', so that U = X_c L1' = X L1' - mu c1 can be
    formed from the raw activations (identical in exact arithmetic).

Output (``linear``):
10. Y = deq(Q(Xt)) deq(Q(R)) + U L2 + mu s   (all float64).
"""
import numpy as np

from . import bf16 as _bf16
from . import lpfit as _lp
from . import mxfp4 as _mx
from . import transforms as _tr


def center(X, on: bool):
    """(mu [M], X_c [M, K]) in float64; mu = 0 when centring is off."""
    X = np.asarray(X, dtype=np.float64)
    if not on:
        return np.zeros(X.shape[0]), X.copy()
    mu = X.mean(axis=1)
    return mu, X - mu[:, None]


def truncated_svd_factors(Wp, r: int):
    """(L1 [K, r], L2 [r, N]) in float64 before rounding: U_r sqrt(S_r), sqrt(S_r) V_r^T,
    plus the full singular value vector."""
    Uf, S, Vt = np.linalg.svd(np.asarray(Wp, dtype=np.float64), full_matrices=False)
    rs = np.sqrt(S[:r])
    return Uf[:, :r] * rs[None, :], rs[:, None] * Vt[:r, :], S


def prepare(W, T: dict, r: int, lp: float | None = None) -> dict:
    """Offline weight preparation (steps 5-9). W: [K, N] (bf16 values as float64 or torch).

    lp: encode the residual with the robust l_p scale fit (``oracle.lpfit``, CentriQ)
    instead of the plain OCP rule; None keeps the plain rule."""
    W = _as_f64(W)
    K, N = W.shape
    s = W.sum(axis=0)
    Wp = _tr.inverse_fold(W, T)
    if r > 0:
        L1u, L2u, S = truncated_svd_factors(Wp, r)
        L1 = _bf16.round_bf16(L1u)
        L2 = _bf16.round_bf16(L2u)
    else:
        S = np.linalg.svd(Wp, compute_uv=False)
        L1 = np.zeros((K, 0))
        L2 = np.zeros((0, N))
    R = Wp - L1 @ L2
    R32 = _bf16.round_f32(R)
    # residual blocks run along K for every output column n: encode R^T [N, K]
    if lp is None:
        r_codes, r_scales = _mx.encode(R32.T)
    else:
        r_codes, r_scales, _ = _lp.encode_lp(R32.T, lp)
    L1p = _tr.forward_fold(L1, T)
    c1 = L1p.sum(axis=0)
    return {"s": s, "Wp": Wp, "L1": L1, "L2": L2, "S": S, "R": R, "R32": R32,
            "r_codes": r_codes, "r_scales": r_scales, "L1p": L1p, "c1": c1,
            "K": K, "N": N, "rank": r}


def quantize_act(X, T: dict, centre_on: bool, prep: dict) -> dict:
    """Online activation half (steps 1-4)."""
    X = _as_f64(X)
    mu, Xc = center(X, centre_on)
    Xt = _tr.apply(Xc, T)
    Xt32 = _bf16.round_f32(Xt)
    codes, scales = _mx.encode(Xt32)
    U = Xt @ prep["L1"]
    return {"mu": mu, "Xc": Xc, "Xt": Xt, "Xt32": Xt32, "codes": codes, "scales": scales,
            "U": U}


def linear_from_parts(act: dict, prep: dict) -> np.ndarray:
    """Step 10 from already-quantized parts."""
    Xq = _mx.decode(act["codes"], act["scales"])
    Rq = _mx.decode(prep["r_codes"], prep["r_scales"]).T          # [K, N]
    Y = Xq @ Rq + act["U"] @ prep["L2"] + np.outer(act["mu"], prep["s"])
    return Y


def linear(X, T: dict, centre_on: bool, prep: dict) -> np.ndarray:
    """Y_ref [M, N] float64 for activations X [M, K]."""
    return linear_from_parts(quantize_act(X, T, centre_on, prep), prep)


def _as_f64(a) -> np.ndarray:
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return a.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a, dtype=np.float64)
