"""The C-ABI library loads and exports every symbol include/kq.h declares; host-side
size queries and argument validation work without a GPU (no compute calls here)."""
import ctypes
import os
import re

import numpy as np
import pytest

import w4a4_post_quantization_token_b200 as kq

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "kq.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kq_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = header_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(kq.lib, n), f"libkq.so does not export {n}"
    assert sorted(kq.SYMBOLS) == names


def test_library_is_in_tree_and_versioned():
    assert os.path.dirname(kq.library_path) == os.path.dirname(kq.__file__)
    assert b"sm_100a" in kq.lib.kq_version()


def test_struct_layout_matches_c():
    # kq_transform_desc: int32 + ptr + int32 + ptr + int32 + ptr + ptr (with padding) = 56
    assert ctypes.sizeof(kq._TransformDesc) == 56
    # + kq_layernorm_desc: int32 + float + ptr + ptr = 24, + int32 codebook (padded to 8)
    assert ctypes.sizeof(kq._LayerDesc) == 16 + 56 + 24 + 8


def _kron():
    return {"kind": "kron", "A": np.eye(4, dtype=np.float32), "B": np.eye(8, dtype=np.float32)}


def test_size_queries():
    L = kq.Layer(1152, 4608, 32, False, {"kind": "rpbh", "perm": np.arange(1152),
                                          "sign": np.ones(1152, np.int8)})
    wb = kq.weights_bytes(L)
    # at least codes + scales + L2^T + L1'^T + sums
    assert wb >= 4608 * 576 + 4608 * 36 + 4608 * 64 * 2 + 144 * 1152 * 2
    for M in (1, 4096, 4097, 35100):
        # codes + scales + fp16 U at least (split-K scratch for small M comes on top)
        assert kq.act_bytes(L, M) >= M * 576 + M * 36 + M * 64 * 2
    assert kq.act_bytes(L, 0) == 0


@pytest.mark.parametrize("K,N,rank,status", [(1000, 64, 0, 2), (64, 40, 0, 2), (64, 64, 65, 2),
                                              (0, 64, 0, 1), (64, 64, -1, 1)])
def test_invalid_shapes_rejected(K, N, rank, status):
    L = kq.Layer(K, N, rank, False, {"kind": "none"})
    assert kq.weights_bytes(L) == 0
    r = kq.lib.kq_quantize_act(L.desc, None, None, 4, None, 0, None)
    assert r == status


def test_invalid_transform_rejected():
    K = 64
    bad_perm = {"kind": "rpbh", "perm": np.zeros(K, np.int32), "sign": np.ones(K, np.int8)}
    assert kq.weights_bytes(kq.Layer(K, 64, 0, False, bad_perm)) == 0
    bad_sign = {"kind": "rpbh", "perm": np.arange(K), "sign": np.zeros(K, np.int8)}
    assert kq.weights_bytes(kq.Layer(K, 64, 0, False, bad_sign)) == 0
    bad_dim = {"kind": "kron", "A": np.eye(2, dtype=np.float32), "B": np.eye(16, dtype=np.float32)}
    assert kq.weights_bytes(kq.Layer(K, 64, 0, False, bad_dim)) == 0
    nan = {"kind": "kron", "A": np.full((4, 4), np.nan, np.float32), "B": np.eye(8, dtype=np.float32)}
    assert kq.weights_bytes(kq.Layer(K, 64, 0, False, nan)) == 0
    assert kq.weights_bytes(kq.Layer(K, 64, 0, False, _kron())) > 0


def test_null_and_alignment_errors_before_any_launch():
    L = kq.Layer(64, 64, 0, False, _kron())
    M = 8
    # null pointers -> invalid argument
    assert kq.lib.kq_linear(L.desc, None, None, M, None, 0, None, 0, None) == 1
    # misaligned device pointers -> alignment error (checked before any CUDA call)
    odd = ctypes.c_void_p(0x1000 + 8)
    ok = ctypes.c_void_p(0x100000)
    assert kq.lib.kq_quantize_act(L.desc, ok, odd, M, ok, 1 << 20, None) == 3
    # a 16-byte boundary is enough (what a TMA global address needs): the call gets past
    # the alignment check and stops at the workspace-size check
    at16 = ctypes.c_void_p(0x1000 + 16)
    assert kq.lib.kq_quantize_act(L.desc, at16, at16, M, at16, 16, None) == 5
    # too-small workspace
    assert kq.lib.kq_quantize_act(L.desc, ok, ok, M, ok, 16, None) == 5
    # bad output dtype
    assert kq.lib.kq_gemm(L.desc, ok, ok, M, ok, 7, None) == 1
    assert kq.lib.kq_debug_encode_f32(ok, M, 33, ok, ok, None) == 2


def test_smooth_quantize_rejects_layers_with_a_transform():
    ok = ctypes.c_void_p(0x100000)
    L = kq.Layer(64, 64, 0, False, _kron())
    assert kq.lib.kq_smooth_quantize_act(L.desc, ok, ok, 8, ok, 1 << 20, None) == 1
    Lc = kq.Layer(64, 64, 0, True, {"kind": "none"})
    assert kq.lib.kq_smooth_quantize_act(Lc.desc, ok, ok, 8, ok, 1 << 20, None) == 1
    L0 = kq.Layer(64, 64, 0, False, {"kind": "none"})
    assert kq.lib.kq_smooth_quantize_act(L0.desc, None, ok, 8, ok, 1 << 20, None) == 1
    assert kq.lib.kq_smooth_quantize_act(L0.desc, ok, ok, 8, ok, 16, None) == 5


def test_lp_entry_points_reject_bad_p():
    ok = ctypes.c_void_p(0x100000)
    L = kq.Layer(64, 64, 0, False, _kron())
    for p in (0.0, -1.0, 2.5, float("nan")):
        assert kq.lib.kq_prepare_weights_lp(L.desc, p, ok, ok, ok, 1 << 30, None) == 1
        assert kq.lib.kq_debug_encode_lp_f32(ok, 8, 64, p, ok, ok, None) == 1


def test_status_strings():
    for s in range(10):
        assert kq.status_string(s)
    assert "timed out" in kq.status_string(kq.ERR_DEVICE_TIMEOUT)
    assert "fp16 range" in kq.status_string(kq.ERR_LOWRANK_RANGE)
    assert "16-byte" in kq.status_string(3)


def test_wait_timeout_entry_validates_before_launch():
    """The bounded-wait exercise takes a limit of 1 us .. 1 s and an aligned workspace;
    anything else is refused on the host."""
    L = kq.Layer(64, 64, 0, False, _kron())
    ok = ctypes.c_void_p(0x100000)
    assert kq.lib.kq_debug_wait_timeout(L.desc, ok, 8, 0, None) == 1
    assert kq.lib.kq_debug_wait_timeout(L.desc, ok, 8, 1000001, None) == 1
    assert kq.lib.kq_debug_wait_timeout(L.desc, None, 8, 1000, None) == 1
    assert kq.lib.kq_debug_wait_timeout(L.desc, ok, 0, 1000, None) == 1
    assert kq.lib.kq_debug_wait_timeout(L.desc, ctypes.c_void_p(0x1000 + 8), 8, 1000, None) == 3


def _ln(K, **kw):
    d = {"gamma": np.ones(K, np.float32), "beta": np.zeros(K, np.float32), "eps": 1e-6}
    d.update(kw)
    return d


def test_layernorm_descriptor_validation():
    K, N = 64, 64
    plain = kq.Layer(K, N, 8, True, _kron())
    ln = kq.Layer(K, N, 8, True, _kron(), layernorm=_ln(K))
    # the front-end adds gamma, beta, the kernel table, diag(gamma) L1' and two sums
    assert kq.weights_bytes(ln) >= kq.weights_bytes(plain) + 8 * K + 12 * K + 2 * 64 * K * 2
    # and two per-token floats to the activations
    assert kq.act_bytes(ln, 300) >= kq.act_bytes(plain, 300) + 2 * 384 * 4
    # it normalises and then centres: centring must be on; eps must be positive and finite
    assert kq.weights_bytes(kq.Layer(K, N, 8, False, _kron(), layernorm=_ln(K))) == 0
    for eps in (0.0, -1e-6, float("nan"), float("inf")):
        assert kq.weights_bytes(kq.Layer(K, N, 8, True, _kron(), layernorm=_ln(K, eps=eps))) == 0
    # gamma / beta are read (and checked) only where they are written into the weights
    ok = ctypes.c_void_p(0x100000)
    bad = kq.Layer(K, N, 8, True, _kron(), layernorm=_ln(K, gamma=np.full(K, np.nan, np.float32)))
    assert kq.weights_bytes(bad) > 0
    assert kq.lib.kq_prepare_weights(bad.desc, ok, ok, ok, 1 << 30, None) == 1
    assert kq.lib.kq_weights_pack(bad.desc, ok, ok, ok, ok, ok, ok, None) == 1
    # the SmoothQuant comparator has no front-end
    L0 = kq.Layer(K, N, 0, True, {"kind": "none"}, layernorm=_ln(K))
    assert kq.lib.kq_smooth_quantize_act(L0.desc, ok, ok, 8, ok, 1 << 20, None) == 1


def _rpbh(K):
    return {"kind": "rpbh", "perm": np.arange(K)[::-1].copy(), "sign": np.ones(K, np.int8)}


def test_codebook_descriptor_validation():
    K, N = 256, 128
    plain = kq.Layer(K, N, 16, True, _rpbh(K))
    lut = kq.Layer(K, N, 16, True, _rpbh(K), codebook="lloydmax")
    # the decoded fp16 residual rides along with the weights; the activation operand is
    # fp16 (2 bytes per element) with one sigma per token and no block scales
    assert kq.weights_bytes(lut) >= kq.weights_bytes(plain) + N * K * 2
    assert kq.act_bytes(lut, 300) >= 300 * K * 2 + 384 * 4
    assert kq.weights_bytes(kq.Layer(K, N, 0, False, {"kind": "none"}, codebook="lloydmax")) > 0
    # designed for the RPBH coordinates: not with the Kronecker transform, not behind the
    # LayerNorm front-end
    assert kq.weights_bytes(kq.Layer(K, N, 16, True, _kron(), codebook="lloydmax")) == 0
    ln = {"gamma": np.ones(K, np.float32), "beta": np.zeros(K, np.float32), "eps": 1e-6}
    assert kq.weights_bytes(kq.Layer(K, N, 16, True, _rpbh(K), layernorm=ln, codebook="lloydmax")) == 0
    bad = kq.Layer(K, N, 16, True, _rpbh(K))
    bad._desc.codebook = 2
    assert kq.weights_bytes(bad) == 0


def test_library_codebook_matches_the_oracle():
    """The library computes its Lloyd-Max codebook with its own host code; it must be the
    oracle's fixed point to float64 rounding."""
    from oracle import lloydmax as lm
    lv, th = kq.lloydmax_codebook()
    pos, pth = lm.magnitudes()
    np.testing.assert_allclose(lv, pos, rtol=1e-13, atol=0)
    np.testing.assert_allclose(th, pth, rtol=1e-13, atol=0)


def test_rpbh_largest_k():
    """The RPBH gather table holds 16-bit byte offsets into a staged row: K <= 32736."""
    ok = kq.Layer(32736, 64, 0, False, _rpbh(32736))
    assert kq.weights_bytes(ok) > 0
    big = kq.Layer(32768, 64, 0, False, _rpbh(32768))
    assert kq.weights_bytes(big) == 0
    assert kq.lib.kq_quantize_act(big.desc, None, None, 4, None, 0, None) == 2


def test_binding_fails_loudly_without_the_library():
    """The product path has no fallback: without libkq.so next to it the package does not
    import (executed here from its source with a location that holds no library)."""
    import types
    src_path = os.path.join(os.path.dirname(kq.__file__), "__init__.py")
    mod = types.ModuleType("kq_without_library")
    mod.__file__ = os.path.join(os.path.dirname(kq.__file__), "no_such_dir", "__init__.py")
    with pytest.raises(ImportError, match="libkq.so not found"):
        exec(compile(open(src_path).read(), mod.__file__, "exec"), mod.__dict__)
