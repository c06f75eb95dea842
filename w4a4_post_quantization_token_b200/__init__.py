"""Python binding of libkq, the B200 (sm_100a) W4A4 quantized linear layer.

Argument marshalling only: every step of the layer runs in the CUDA library
(include/kq.h); this module checks tensor placement, dtypes and sizes, passes raw
device pointers and the current CUDA stream, and raises on a non-OK status.
PyTorch is used for device memory and streams. There is no CPU fallback: if the
shared library is missing or cannot be loaded, importing this package raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

__all__ = ["KQError", "Layer", "lib", "library_path", "weights_bytes", "act_bytes",
           "prepare_ws_bytes", "prepare_weights", "prepare_weights_lp", "debug_encode_lp_f32", "quantize_act", "smooth_quantize_act", "linear",
           "linear_noalloc", "lloydmax_codebook", "CB_MXFP4", "CB_LLOYDMAX",
           "linear_host", "NOALLOC_WORKSPACE_BYTES",
           "gemm", "weights_pack", "weights_unpack", "act_pack", "act_unpack",
           "debug_transform", "debug_encode_f32", "debug_wait_timeout", "last_device_error",
           "status_string", "ERR_DEVICE_TIMEOUT", "ERR_LOWRANK_RANGE",
           "OUT_F32", "OUT_BF16", "SYMBOLS"]

OUT_F32, OUT_BF16 = 0, 1
ERR_DEVICE_TIMEOUT, ERR_LOWRANK_RANGE = 7, 9
T_NONE, T_KRON, T_RPBH = 0, 1, 2
_KIND = {"none": T_NONE, "kron": T_KRON, "rpbh": T_RPBH}
CB_MXFP4, CB_LLOYDMAX = 0, 1
_CODEBOOK = {"mxfp4": CB_MXFP4, "lloydmax": CB_LLOYDMAX}

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libkq.so")

# every symbol include/kq.h declares
SYMBOLS = ["kq_weights_bytes", "kq_act_bytes", "kq_prepare_ws_bytes", "kq_prepare_weights",
           "kq_quantize_act", "kq_linear", "kq_linear_host", "kq_gemm", "kq_weights_pack",
           "kq_weights_unpack", "kq_act_pack", "kq_act_unpack", "kq_debug_transform",
           "kq_debug_encode_f32", "kq_last_device_error", "kq_status_string", "kq_version",
           "kq_linear_noalloc", "kq_smooth_quantize_act", "kq_prepare_weights_lp",
           "kq_debug_encode_lp_f32", "kq_lloydmax_codebook", "kq_debug_wait_timeout"]


class KQError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


if not os.path.exists(library_path):
    raise ImportError(f"libkq.so not found at {library_path}; build it with "
                      "`python w4a4_post_quantization_token_b200/build.py`")
lib = ctypes.CDLL(library_path)


class _TransformDesc(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("A", ctypes.POINTER(ctypes.c_float)),
                ("a_dim", ctypes.c_int32), ("B", ctypes.POINTER(ctypes.c_float)),
                ("b_dim", ctypes.c_int32), ("perm", ctypes.POINTER(ctypes.c_int32)),
                ("sign", ctypes.POINTER(ctypes.c_int8))]


class _LayerNormDesc(ctypes.Structure):
    _fields_ = [("on", ctypes.c_int32), ("eps", ctypes.c_float),
                ("gamma", ctypes.POINTER(ctypes.c_float)), ("beta", ctypes.POINTER(ctypes.c_float))]


class _LayerDesc(ctypes.Structure):
    _fields_ = [("K", ctypes.c_int32), ("N", ctypes.c_int32), ("rank", ctypes.c_int32),
                ("center", ctypes.c_int32), ("t", _TransformDesc), ("ln", _LayerNormDesc),
                ("codebook", ctypes.c_int32)]


_P = ctypes.c_void_p
_D = ctypes.POINTER(_LayerDesc)
_sigs = {
    "kq_weights_bytes": (ctypes.c_size_t, [_D]),
    "kq_act_bytes": (ctypes.c_size_t, [_D, ctypes.c_int32]),
    "kq_prepare_ws_bytes": (ctypes.c_size_t, [_D]),
    "kq_prepare_weights": (ctypes.c_int, [_D, _P, _P, _P, ctypes.c_size_t, _P]),
    "kq_quantize_act": (ctypes.c_int, [_D, _P, _P, ctypes.c_int32, _P, ctypes.c_size_t, _P]),
    "kq_linear": (ctypes.c_int, [_D, _P, _P, ctypes.c_int32, _P, ctypes.c_int32, _P,
                                 ctypes.c_size_t, _P]),
    "kq_prepare_weights_lp": (ctypes.c_int, [_D, ctypes.c_double, _P, _P, _P, ctypes.c_size_t, _P]),
    "kq_debug_encode_lp_f32": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_int32, ctypes.c_double,
                                              _P, _P, _P]),
    "kq_smooth_quantize_act": (ctypes.c_int, [_D, _P, _P, ctypes.c_int32, _P, ctypes.c_size_t, _P]),
    "kq_linear_noalloc": (ctypes.c_int, [_D, _P, _P, ctypes.c_int32, _P, ctypes.c_int32, _P]),
    "kq_linear_host": (ctypes.c_int, [_D, _P, _P, _P, ctypes.c_int32, _P, _P, ctypes.c_int32,
                                      _P, ctypes.c_size_t, _P]),
    "kq_gemm": (ctypes.c_int, [_D, _P, _P, ctypes.c_int32, _P, ctypes.c_int32, _P]),
    "kq_weights_pack": (ctypes.c_int, [_D, _P, _P, _P, _P, _P, _P, _P]),
    "kq_weights_unpack": (ctypes.c_int, [_D, _P, _P, _P, _P, _P, _P, _P, _P]),
    "kq_act_pack": (ctypes.c_int, [_D, _P, _P, _P, _P, ctypes.c_int32, _P, ctypes.c_size_t, _P]),
    "kq_act_unpack": (ctypes.c_int, [_D, _P, ctypes.c_int32, _P, _P, _P, _P, _P]),
    "kq_debug_transform": (ctypes.c_int, [_D, _P, _P, ctypes.c_int32, _P, _P, _P]),
    "kq_debug_encode_f32": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_int32, _P, _P, _P]),
    "kq_last_device_error": (ctypes.c_int, [_D, _P, ctypes.c_int32, _P]),
    "kq_debug_wait_timeout": (ctypes.c_int, [_D, _P, ctypes.c_int32, ctypes.c_uint32, _P]),
    "kq_lloydmax_codebook": (ctypes.c_int, [_P, _P]),
    "kq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "kq_version": (ctypes.c_char_p, []),
}
for _name, (_res, _args) in _sigs.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def lloydmax_codebook() -> tuple[np.ndarray, np.ndarray]:
    """The library's (8 positive levels, 7 thresholds) of its 16-level Lloyd-Max codebook."""
    lv = np.zeros(8, np.float64)
    th = np.zeros(7, np.float64)
    _check(lib.kq_lloydmax_codebook(lv.ctypes.data_as(_P), th.ctypes.data_as(_P)),
           "kq_lloydmax_codebook")
    return lv, th


def status_string(s: int) -> str:
    return lib.kq_status_string(int(s)).decode()


def _check(status: int, where: str) -> None:
    if status != 0:
        raise KQError(status, where)


class Layer:
    """Host description of one linear layer (the C ``kq_layer_desc``).

    ``transform`` is ``{"kind": "kron", "A": 4x4, "B": 8x8}``,
    ``{"kind": "rpbh", "perm": int[K], "sign": +-1[K]}`` or ``{"kind": "none"}``.
    ``layernorm`` (optional) is ``{"gamma": float[K], "beta": float[K], "eps": float}``: the
    fused LayerNorm front-end (needs ``center``).
    ``codebook`` is ``"mxfp4"`` (default) or ``"lloydmax"``: the 16-level Lloyd-Max
    codebook with a per-token sigma (RPBH or no transform; activations reach the fp16
    tensor-core GEMM as decoded fp16 values).
    The host arrays are kept alive by this object."""

    def __init__(self, K: int, N: int, rank: int, center: bool, transform: dict,
                 layernorm: dict | None = None, codebook: str = "mxfp4"):
        self.K, self.N, self.rank, self.center = int(K), int(N), int(rank), bool(center)
        self.transform = transform
        kind = _KIND[transform["kind"]]
        t = _TransformDesc(kind=kind)
        self._keep = []
        if kind == T_KRON:
            A = np.ascontiguousarray(transform["A"], dtype=np.float32)
            B = np.ascontiguousarray(transform["B"], dtype=np.float32)
            self._keep += [A, B]
            t.A = A.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
            t.B = B.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
            t.a_dim, t.b_dim = A.shape[0], B.shape[0]
        elif kind == T_RPBH:
            perm = np.ascontiguousarray(transform["perm"], dtype=np.int32)
            sign = np.ascontiguousarray(transform["sign"], dtype=np.int8)
            self._keep += [perm, sign]
            t.perm = perm.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
            t.sign = sign.ctypes.data_as(ctypes.POINTER(ctypes.c_int8))
        ln = _LayerNormDesc(on=0)
        self.layernorm = layernorm
        if layernorm is not None:
            g = np.ascontiguousarray(layernorm["gamma"], dtype=np.float32)
            b = np.ascontiguousarray(layernorm["beta"], dtype=np.float32)
            self._keep += [g, b]
            ln.on, ln.eps = 1, float(layernorm.get("eps", 1e-6))
            ln.gamma = g.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
            ln.beta = b.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
        self.codebook = codebook
        self._desc = _LayerDesc(K=self.K, N=self.N, rank=self.rank, center=int(self.center), t=t,
                                ln=ln, codebook=_CODEBOOK[codebook])

    @property
    def desc(self):
        return ctypes.byref(self._desc)


def _ptr(t) -> int | None:
    return None if t is None else int(t.data_ptr())


def _stream(stream=None) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _need(t, dtype, numel: int | None = None, name: str = "tensor", cuda: bool = True):
    import torch
    if t is None:
        raise ValueError(f"{name} is required")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name} has {t.numel()} elements, needs {numel}")
    return t


def weights_bytes(layer: Layer) -> int:
    return int(lib.kq_weights_bytes(layer.desc))


def act_bytes(layer: Layer, M: int) -> int:
    return int(lib.kq_act_bytes(layer.desc, int(M)))


def prepare_ws_bytes(layer: Layer) -> int:
    return int(lib.kq_prepare_ws_bytes(layer.desc))


def prepare_weights(layer: Layer, W, weights, ws, stream=None) -> None:
    import torch
    _need(W, torch.bfloat16, layer.K * layer.N, "W")
    _need(weights, torch.uint8, weights_bytes(layer), "weights")
    _need(ws, torch.uint8, None, "ws")
    _check(lib.kq_prepare_weights(layer.desc, _ptr(W), _ptr(weights), _ptr(ws), ws.numel(),
                                  _stream(stream)), "kq_prepare_weights")


def quantize_act(layer: Layer, weights, X, act, stream=None) -> None:
    import torch
    M = X.shape[0]
    _need(X, torch.bfloat16, M * layer.K, "X")
    _need(act, torch.uint8, act_bytes(layer, M), "act")
    _check(lib.kq_quantize_act(layer.desc, _ptr(weights), _ptr(X), M, _ptr(act), act.numel(),
                               _stream(stream)), "kq_quantize_act")


def prepare_weights_lp(layer: Layer, p: float, W, weights, ws, stream=None) -> None:
    """prepare_weights with the robust l_p fit of the residual's block scales."""
    import torch
    _need(W, torch.bfloat16, layer.K * layer.N, "W")
    _need(weights, torch.uint8, weights_bytes(layer), "weights")
    _need(ws, torch.uint8, None, "ws")
    _check(lib.kq_prepare_weights_lp(layer.desc, float(p), _ptr(W), _ptr(weights), _ptr(ws),
                                     ws.numel(), _stream(stream)), "kq_prepare_weights_lp")


def debug_encode_lp_f32(V, p: float, codes, scales, stream=None) -> None:
    M, K = V.shape
    _check(lib.kq_debug_encode_lp_f32(_ptr(V), M, K, float(p), _ptr(codes), _ptr(scales),
                                      _stream(stream)), "kq_debug_encode_lp_f32")


def smooth_quantize_act(layer: Layer, inv_s, X, act, stream=None) -> None:
    """SmoothQuant comparator: per-channel multiply by inv_s (fp32 [K]), then MXFP4."""
    import torch
    M = X.shape[0]
    _need(inv_s, torch.float32, layer.K, "inv_s")
    _need(X, torch.bfloat16, M * layer.K, "X")
    _need(act, torch.uint8, act_bytes(layer, M), "act")
    _check(lib.kq_smooth_quantize_act(layer.desc, _ptr(inv_s), _ptr(X), M, _ptr(act), act.numel(),
                                      _stream(stream)), "kq_smooth_quantize_act")


def linear(layer: Layer, weights, X, Y, act, out_dtype: int = OUT_F32, stream=None) -> None:
    import torch
    M = X.shape[0]
    _need(X, torch.bfloat16, M * layer.K, "X")
    _need(Y, torch.bfloat16 if out_dtype == OUT_BF16 else torch.float32, M * layer.N, "Y")
    _need(act, torch.uint8, act_bytes(layer, M), "act")
    _check(lib.kq_linear(layer.desc, _ptr(weights), _ptr(X), M, _ptr(Y), int(out_dtype), _ptr(act),
                         act.numel(), _stream(stream)), "kq_linear")


def linear_noalloc(layer: Layer, weights, X, Y, out_dtype: int = OUT_F32, stream=None) -> None:
    """kq_linear on the library's built-in workspace: no workspace argument, nothing
    allocated. Calls that can overlap on the GPU share that workspace and race."""
    import torch
    M = X.shape[0]
    _need(X, torch.bfloat16, M * layer.K, "X")
    _need(Y, torch.bfloat16 if out_dtype == OUT_BF16 else torch.float32, M * layer.N, "Y")
    _check(lib.kq_linear_noalloc(layer.desc, _ptr(weights), _ptr(X), M, _ptr(Y), int(out_dtype),
                                 _stream(stream)), "kq_linear_noalloc")


NOALLOC_WORKSPACE_BYTES = 16 << 20


def linear_host(layer: Layer, weights, X_host, X_dev, Y_host, Y_dev, act,
                out_dtype: int = OUT_F32, stream=None) -> None:
    """Host-buffer variant: X_host and Y_host are pinned CPU tensors."""
    import torch
    M = X_host.shape[0]
    _need(X_host, torch.bfloat16, M * layer.K, "X_host", cuda=False)
    _need(X_dev, torch.bfloat16, M * layer.K, "X_dev")
    ydt = torch.bfloat16 if out_dtype == OUT_BF16 else torch.float32
    _need(Y_host, ydt, M * layer.N, "Y_host", cuda=False)
    _need(Y_dev, ydt, M * layer.N, "Y_dev")
    _check(lib.kq_linear_host(layer.desc, _ptr(weights), _ptr(X_host), _ptr(X_dev), M,
                              _ptr(Y_host), _ptr(Y_dev), int(out_dtype), _ptr(act), act.numel(),
                              _stream(stream)), "kq_linear_host")


def gemm(layer: Layer, weights, act, M: int, Y, out_dtype: int = OUT_F32, stream=None) -> None:
    _check(lib.kq_gemm(layer.desc, _ptr(weights), _ptr(act), int(M), _ptr(Y), int(out_dtype),
                       _stream(stream)), "kq_gemm")


def weights_pack(layer: Layer, r_codes, r_scales, L1p, L2, s, weights, stream=None) -> None:
    import torch
    _need(r_codes, torch.uint8, layer.N * layer.K // 2, "r_codes")
    _need(r_scales, torch.uint8, layer.N * layer.K // 32, "r_scales")
    _need(s, torch.float32, layer.N, "s")
    if layer.rank:
        _need(L1p, torch.float32, layer.K * layer.rank, "L1p")
        _need(L2, torch.bfloat16, layer.rank * layer.N, "L2")
    _need(weights, torch.uint8, weights_bytes(layer), "weights")
    _check(lib.kq_weights_pack(layer.desc, _ptr(r_codes), _ptr(r_scales), _ptr(L1p), _ptr(L2),
                               _ptr(s), _ptr(weights), _stream(stream)), "kq_weights_pack")


def weights_unpack(layer: Layer, weights, r_codes=None, r_scales=None, L1p=None, L2=None, c1=None,
                   s=None, stream=None) -> None:
    _check(lib.kq_weights_unpack(layer.desc, _ptr(weights), _ptr(r_codes), _ptr(r_scales),
                                 _ptr(L1p), _ptr(L2), _ptr(c1), _ptr(s), _stream(stream)),
           "kq_weights_unpack")


def act_pack(layer: Layer, codes, scales, mu, U, M: int, act, stream=None) -> None:
    _check(lib.kq_act_pack(layer.desc, _ptr(codes), _ptr(scales), _ptr(mu), _ptr(U), int(M),
                           _ptr(act), act.numel(), _stream(stream)), "kq_act_pack")


def act_unpack(layer: Layer, act, M: int, codes=None, scales=None, mu=None, U=None,
               stream=None) -> None:
    _check(lib.kq_act_unpack(layer.desc, _ptr(act), int(M), _ptr(codes), _ptr(scales), _ptr(mu),
                             _ptr(U), _stream(stream)), "kq_act_unpack")


def debug_transform(layer: Layer, weights, X, Xt, mu, stream=None) -> None:
    _check(lib.kq_debug_transform(layer.desc, _ptr(weights), _ptr(X), X.shape[0], _ptr(Xt),
                                  _ptr(mu), _stream(stream)), "kq_debug_transform")


def debug_encode_f32(V, codes, scales, stream=None) -> None:
    M, K = V.shape
    _check(lib.kq_debug_encode_f32(_ptr(V), M, K, _ptr(codes), _ptr(scales), _stream(stream)),
           "kq_debug_encode_f32")


def last_device_error(layer: Layer, act, M: int, stream=None) -> int:
    """0 if the device error word is clear, else ERR_DEVICE_TIMEOUT (a bounded device wait
    ran out) or ERR_LOWRANK_RANGE (a low-rank activation was saturated to the fp16 range).
    Synchronises the stream and clears the word."""
    return int(lib.kq_last_device_error(layer.desc, _ptr(act), int(M), _stream(stream)))


def debug_wait_timeout(layer: Layer, act, M: int, limit_us: int, stream=None) -> None:
    """Enqueue one warp that waits limit_us on a barrier nothing completes, so that the
    next last_device_error on `act` reports ERR_DEVICE_TIMEOUT."""
    _need(act, __import__("torch").uint8, act_bytes(layer, M), "act")
    _check(lib.kq_debug_wait_timeout(layer.desc, _ptr(act), int(M), int(limit_us), _stream(stream)),
           "kq_debug_wait_timeout")
