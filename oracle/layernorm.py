"""LayerNorm front-end fused with the W4A4 layer's online half (oracle, test infrastructure).

The KroQuant commentary (section 01) says the online transform cannot be folded away
because normalisation layers sit between the blocks. This front-end applies that
normalisation in the same pass: per token, LayerNorm over the K channels with a per-channel
affine, then the layer as before (CentriQ centring of the normalised token, block
transform, MXFP4, low-rank branch).

Readings (the pages name LayerNorm but give no formula): the usual one,
    y = (x - m) / sqrt(v + eps) * gamma + beta,
m = mean_k x, v = mean_k (x - m)^2 (biased), gamma and beta per channel (fixed per layer).
Per-sample adaLN modulation vectors are outside this front-end (a caller folds one
sample's vectors into gamma and beta, or calls once per sample).
"""
import numpy as np


def stats(X, eps: float):
    """Per-token mean m [M] and reciprocal standard deviation rstd [M] (float64)."""
    X = np.asarray(X, dtype=np.float64)
    m = X.mean(axis=1)
    v = ((X - m[:, None]) ** 2).mean(axis=1)
    return m, 1.0 / np.sqrt(v + eps)


def layernorm(X, gamma, beta, eps: float) -> np.ndarray:
    """y [M, K] float64."""
    X = np.asarray(X, dtype=np.float64)
    m, rstd = stats(X, eps)
    g = np.asarray(gamma, dtype=np.float64)
    b = np.asarray(beta, dtype=np.float64)
    return (X - m[:, None]) * rstd[:, None] * g[None, :] + b[None, :]


def lowrank_input_parts(X, gamma, beta, eps: float, L1p):
    """The decomposition the low-rank kernel uses to form y L1' from raw x:
    y L1' = rstd * (x (diag(gamma) L1')) - rstd * m * (gamma^T L1') + beta^T L1'.
    Returns (direct y L1', decomposed value) for a test to compare."""
    X = np.asarray(X, dtype=np.float64)
    g = np.asarray(gamma, dtype=np.float64)
    b = np.asarray(beta, dtype=np.float64)
    L1p = np.asarray(L1p, dtype=np.float64)
    m, rstd = stats(X, eps)
    direct = layernorm(X, g, b, eps) @ L1p
    L1g = g[:, None] * L1p
    decomposed = (rstd[:, None] * (X @ L1g) - (rstd * m)[:, None] * (g @ L1p)[None, :]
                  + (b @ L1p)[None, :])
    return direct, decomposed
