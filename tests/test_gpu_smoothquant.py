"""GPU: the SmoothQuant comparator (kq_smooth_quantize_act) against the oracle.

The kernel multiplies each bf16 element by the fp32 inverse channel scale and encodes
the fp32 product, exactly as the oracle does, so codes and scales are compared bit for
bit (several tiles, ragged M, K from 64 to 12288). The whole SmoothQuant W4A4 layer then
runs through the unchanged FP4 GEMM with diag(s) W prepared by the oracle; both operands
are identical, so the output differs from the fp64 oracle only by fp32 accumulation."""
import numpy as np
import pytest

from oracle import smoothquant as sq
from synthetic import make_inputs, workload
from tests.kqtest import pack_nibbles, rel_fro, unpack_nibbles

pytestmark = pytest.mark.gpu


def _case(index, **kw):
    w = workload(index, **kw)
    inp = make_inputs(w)
    X = inp["X"].float().numpy().astype(np.float64)
    W = inp["W"].float().numpy().astype(np.float64)
    s = sq.scales_from(X, W, alpha=0.5)
    return w, inp, X, W, s


def _quantize(w, inp, inv32):
    import torch
    import w4a4_post_quantization_token_b200 as kq
    L = kq.Layer(w.K, w.N, 0, False, {"kind": "none"})
    act = torch.empty(kq.act_bytes(L, w.M), dtype=torch.uint8, device="cuda")
    kq.smooth_quantize_act(L, torch.from_numpy(inv32).cuda(), inp["X"].cuda(), act)
    codes = torch.empty((w.M, w.K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((w.M, w.K // 32), dtype=torch.uint8, device="cuda")
    mu = torch.empty(w.M, dtype=torch.float32, device="cuda")
    kq.act_unpack(L, act, w.M, codes, scales, mu)
    torch.cuda.synchronize()
    assert kq.last_device_error(L, act, w.M) == 0
    return L, act, unpack_nibbles(codes.cpu().numpy()), scales.cpu().numpy(), mu.cpu().numpy()


@pytest.mark.parametrize("index,kw", [(2, dict(M=300, N=256)), (3, dict(M=129, N=256)),
                                      (4, dict(M=65, N=256)), (1, dict(M=1, N=256)),
                                      (3, dict(M=200, K=64, N=256))],
                         ids=["K1152", "K3072", "K12288", "M1", "K64"])
def test_codes_and_scales_bit_exact(cuda_device, index, kw):
    w, inp, X, W, s = _case(index, **kw)
    inv32 = sq.inverse_scales_f32(s)
    ref = sq.quantize_act(X, inv32)
    _, _, codes, scales, mu = _quantize(w, inp, inv32)
    np.testing.assert_array_equal(scales, ref["scales"])
    np.testing.assert_array_equal(codes, ref["codes"])
    assert np.all(mu == 0)


def test_smoothquant_layer(cuda_device):
    import torch
    import w4a4_post_quantization_token_b200 as kq
    w, inp, X, W, s = _case(2, M=300, N=512)
    inv32 = sq.inverse_scales_f32(s)
    prep = sq.prepare(W, s)
    L, act, _, _, _ = _quantize(w, inp, inv32)
    wbuf = torch.empty(kq.weights_bytes(L), dtype=torch.uint8, device="cuda")
    kq.weights_pack(L, torch.from_numpy(pack_nibbles(prep["r_codes"])).cuda(),
                    torch.from_numpy(np.ascontiguousarray(prep["r_scales"])).cuda(), None, None,
                    torch.zeros(w.N, dtype=torch.float32).cuda(), wbuf)
    Y = torch.empty((w.M, w.N), dtype=torch.float32, device="cuda")
    kq.gemm(L, wbuf, act, w.M, Y)
    torch.cuda.synchronize()
    Yref = sq.linear(X, inv32, prep)
    assert rel_fro(Y.cpu().double().numpy(), Yref) <= 1e-5
    # and the method's own error against the unquantised product, for the record
    assert rel_fro(Yref, X @ W) < 0.5
