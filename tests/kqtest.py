"""Test helpers: canonical-layout packing (as include/kq.h defines it), cached oracle
preparation, and moving oracle-prepared weights into the library's buffer through
its own kq_weights_pack. Nothing here computes any part of the layer."""
from __future__ import annotations

import functools

import numpy as np

from oracle import layer as olayer
from synthetic import make_inputs, workload


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """uint8 codes [rows, K] (0..15) -> canonical [rows, K/2], element 2j in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return np.ascontiguousarray((c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8))


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 15
    out[:, 1::2] = p >> 4
    return out


@functools.lru_cache(maxsize=None)
def inputs_and_prep(index: int, **kw):
    w = workload(index, **kw)
    inp = make_inputs(w)
    prep = olayer.prepare(inp["W"], inp["T"], w.rank)
    return w, inp, prep


def cached(index: int, M=None, K=None, N=None, rank=None):
    kw = {}
    for k, v in (("M", M), ("K", K), ("N", N), ("rank", rank)):
        if v is not None:
            kw[k] = v
    return inputs_and_prep(index, **kw)


def make_layer(w, T):
    import w4a4_post_quantization_token_b200 as kq
    return kq.Layer(w.K, w.N, w.rank, w.center, T)


def torch_bf16_bits_to_tensor(a_f64: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a_f64, dtype=np.float32)).to(torch.bfloat16)


def pack_oracle_weights(layer, prep, device="cuda"):
    """Prepared-weights buffer filled from the oracle's canonical parts via kq_weights_pack."""
    import torch
    import w4a4_post_quantization_token_b200 as kq
    K, N, r = layer.K, layer.N, layer.rank
    rc = torch.from_numpy(pack_nibbles(prep["r_codes"])).to(device)
    rs = torch.from_numpy(np.ascontiguousarray(prep["r_scales"])).to(device)
    s = torch.from_numpy(prep["s"].astype(np.float32)).to(device)
    if r:
        L1p = torch.from_numpy(prep["L1p"].astype(np.float32)).to(device).contiguous()
        L2 = torch_bf16_bits_to_tensor(prep["L2"]).to(device).contiguous()
    else:
        L1p = L2 = None
    wbuf = torch.empty(kq.weights_bytes(layer), dtype=torch.uint8, device=device)
    kq.weights_pack(layer, rc, rs, L1p, L2, s, wbuf)
    return wbuf


def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
