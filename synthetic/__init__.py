"""Seeded synthetic workloads for the W4A4 linear layer.

This module only draws random inputs. It holds none of the layer's arithmetic
(no centring, transform, quantisation or contraction), so both the CPU oracle
and the CUDA path can take their inputs from it without sharing any method code.

The five workloads stand in for the models named on the pages (PixArt-Sigma,
FLUX.1, video DiTs). No dataset or trained weight is used: activations follow
the adaLN-style law the workload names (per-token scale and shift, a few fixed
outlier channels), weights are Gaussian, and the transform parameters are drawn
the way the workload describes them.

Recipe (all draws from ``numpy.random.default_rng(seed)`` in the order below):

1. outlier channel indices: ``rng.choice(K, n_outliers, replace=False)``;
2. per-token scale ``a_m`` (``U(lo, hi)``, or 1 when the law has none);
3. per-token shift ``b_m ~ N(0, shift_std)`` (std, not variance);
4. ``z ~ N(0, 1)`` of shape ``[M, K]`` (float32 draws);
5. ``x = z * a_m + b_m`` (or ``GELU(z * gelu_std) + b_m`` for the post-GELU law,
   GELU in its exact erf form), then ``x[:, outliers] *= outlier_factor``;
   X is rounded to bf16;
6. ``W ~ N(0, w_std)`` of shape ``[K, N]``, rounded to bf16;
7. transform: Kronecker factors ``A = I + N(0, 0.1)`` (4x4) and
   ``B = I + N(0, 0.1)`` (8x8), drawn from ``default_rng(seed + 1000 * t)`` for
   attempt ``t = 1, 2, ...`` until both condition numbers are below 100, stored
   as float32; or, for the permuted block-Hadamard transform, a permutation of
   ``[0, K)`` and Rademacher signs from ``default_rng(seed + 1000)``;
8. LayerNorm front-end parameters (only where a case asks for them), from
   ``default_rng(seed + 2000)``: ``gamma = 1 + 0.25 N(0, 1)`` then ``beta = 0.5 N(0, 1)``,
   each ``[K]`` float32, ``eps = 1e-6`` (adaLN-style modulated scale and shift).
"""
from __future__ import annotations

import dataclasses

import numpy as np

__all__ = ["Workload", "WORKLOADS", "workload", "make_activations", "make_weight",
           "make_transform", "make_inputs", "make_layernorm"]


@dataclasses.dataclass(frozen=True)
class Workload:
    index: int              # 1-based workload number
    name: str
    M: int                  # tokens (batch folded in)
    K: int                  # input features
    N: int                  # output features
    transform: str          # "kron" | "rpbh"
    center: bool            # per-token mean centring with rank-1 restore
    rank: int               # low-rank branch rank r
    seed: int
    # activation law
    scale_lo: float | None  # per-token scale U(lo, hi); None -> 1
    scale_hi: float | None
    shift_std: float        # per-token shift N(0, shift_std)
    n_outliers: int
    outlier_factor: float
    gelu_std: float | None  # post-GELU law: GELU(N(0, gelu_std)) + shift
    w_std: float

    @property
    def label(self) -> str:
        return f"{self.name} M={self.M} K={self.K} N={self.N} {self.transform} " \
               f"center={int(self.center)} r={self.rank}"


WORKLOADS = {
    1: Workload(1, "tiny_linear", 256, 1152, 1152, "kron", True, 16, 0,
                None, None, 3.0, 4, 50.0, None, 0.02),
    2: Workload(2, "pixart_sigma_mlp_fc1", 4096, 1152, 4608, "rpbh", False, 32, 1,
                0.5, 2.0, 2.0, 8, 30.0, None, 0.02),
    3: Workload(3, "flux_fused_qkv", 4608, 3072, 9216, "kron", True, 32, 2,
                0.5, 2.0, 2.0, 16, 40.0, None, 0.02),
    4: Workload(4, "flux_mlp_fc2", 4608, 12288, 3072, "rpbh", False, 32, 3,
                None, None, 1.0, 0, 1.0, 1.5, 0.015),
    5: Workload(5, "video_dit_long_seq", 35100, 3072, 3072, "kron", True, 64, 4,
                None, None, 4.0, 16, 50.0, None, 0.02),
}


def workload(index: int, **overrides) -> Workload:
    """Return workload ``index`` (1..5), optionally with fields replaced
    (e.g. ``M=300`` for a reduced-size parity case of the same law)."""
    return dataclasses.replace(WORKLOADS[index], **overrides)


def _to_bf16(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def make_activations(w: Workload):
    """bf16 activations ``[M, K]`` (a torch CPU tensor) and the outlier indices."""
    rng = np.random.default_rng(w.seed)
    outliers = np.sort(rng.choice(w.K, w.n_outliers, replace=False)) if w.n_outliers else \
        np.zeros(0, dtype=np.int64)
    if w.scale_lo is not None:
        a = rng.uniform(w.scale_lo, w.scale_hi, size=(w.M, 1)).astype(np.float32)
    else:
        a = np.ones((w.M, 1), dtype=np.float32)
    b = (rng.standard_normal((w.M, 1)) * w.shift_std).astype(np.float32)
    z = rng.standard_normal((w.M, w.K), dtype=np.float32)
    if w.gelu_std is not None:
        import torch
        t = torch.from_numpy(z) * w.gelu_std
        x = torch.nn.functional.gelu(t, approximate="none").numpy() + b
    else:
        x = z * a + b
    if w.n_outliers:
        x[:, outliers] *= np.float32(w.outlier_factor)
    return _to_bf16(x), outliers


def make_weight(w: Workload):
    """bf16 weight ``[K, N]`` (torch CPU tensor), row-vector convention Y = X W."""
    rng = np.random.default_rng(w.seed + 500)
    W = rng.standard_normal((w.K, w.N), dtype=np.float32) * np.float32(w.w_std)
    return _to_bf16(W)


def make_transform(w: Workload) -> dict:
    """Transform parameters as plain arrays.

    kron: ``{"kind": "kron", "A": float32[4,4], "B": float32[8,8]}``
    rpbh: ``{"kind": "rpbh", "perm": int32[K], "sign": int8[K]}``
    """
    if w.transform == "kron":
        t = 1
        while True:
            rng = np.random.default_rng(w.seed + 1000 * t)
            A = (np.eye(4) + 0.1 * rng.standard_normal((4, 4))).astype(np.float32)
            B = (np.eye(8) + 0.1 * rng.standard_normal((8, 8))).astype(np.float32)
            if np.linalg.cond(A.astype(np.float64)) < 100 and \
               np.linalg.cond(B.astype(np.float64)) < 100:
                return {"kind": "kron", "A": A, "B": B}
            t += 1
    if w.transform == "rpbh":
        rng = np.random.default_rng(w.seed + 1000)
        perm = rng.permutation(w.K).astype(np.int32)
        sign = np.where(rng.integers(0, 2, size=w.K) == 1, 1, -1).astype(np.int8)
        return {"kind": "rpbh", "perm": perm, "sign": sign}
    if w.transform == "none":
        return {"kind": "none"}
    raise ValueError(w.transform)


def make_layernorm(w: Workload) -> dict:
    """``{"gamma": float32[K], "beta": float32[K], "eps": 1e-6}`` (recipe step 8)."""
    rng = np.random.default_rng(w.seed + 2000)
    gamma = (1.0 + 0.25 * rng.standard_normal(w.K)).astype(np.float32)
    beta = (0.5 * rng.standard_normal(w.K)).astype(np.float32)
    return {"gamma": gamma, "beta": beta, "eps": 1e-6}


def make_inputs(w: Workload) -> dict:
    X, outliers = make_activations(w)
    return {"X": X, "W": make_weight(w), "T": make_transform(w), "outliers": outliers,
            "workload": w}


def exact_grid_inputs(M: int, K: int, N: int, seed: int):
    """Inputs whose MXFP4 encoding is exact: every 32-element block holds values
    ``g * 2^s`` with ``g`` on the E2M1 grid and one power of two ``s`` per block,
    and every block contains a +-6 so that its shared scale is exactly ``2^s``.
    Returned as float32 arrays ``Xq [M, K]`` and ``Wq [N, K]`` (K-major rows).
    Used to check GEMM layouts: the fp64 product of such inputs is exact."""
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    rng = np.random.default_rng(seed)

    def one(rows):
        g = grid[rng.integers(0, 8, size=(rows, K))] * np.where(
            rng.integers(0, 2, size=(rows, K)) == 1, -1.0, 1.0)
        blk = g.reshape(rows, K // 32, 32)
        pos = rng.integers(0, 32, size=(rows, K // 32))
        np.put_along_axis(blk, pos[..., None], 6.0 * np.where(
            rng.integers(0, 2, size=(rows, K // 32, 1)) == 1, -1.0, 1.0), axis=2)
        s = rng.integers(-6, 4, size=(rows, K // 32, 1)).astype(np.float64)
        return (blk * np.exp2(s)).reshape(rows, K).astype(np.float32)

    return one(M), one(N)

