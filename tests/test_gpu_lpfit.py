"""GPU: the robust l_p block-scale fit (CentriQ) against the oracle.

The device encoder and the oracle evaluate the same candidate exponents with the same
rounding; the l_p objectives are float64 sums in different orders (and pow from two
libraries), so a block may choose differently only where its two best candidates are
within 1e-12 (relative) of each other. Where the scale agrees the codes must agree bit for
bit. The whole layer prepared with kq_prepare_weights_lp must match the oracle's layer
with the same fit within the layer tolerance."""
import numpy as np
import pytest

from oracle import layer as olayer
from oracle import lpfit
from synthetic import make_inputs, workload
from tests.kqtest import make_layer, rel_fro, unpack_nibbles

pytestmark = pytest.mark.gpu


def _rows(seed, M=96, K=1152):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((M, K))
    v[rng.random((M, K)) < 0.03] *= 30.0
    v[: M // 4] *= 2.0 ** rng.integers(-20, 20, (M // 4, 1))
    return v.astype(np.float32)


@pytest.mark.parametrize("p", [0.5, 1.0, 2.0])
def test_debug_encoder_matches_oracle(cuda_device, p):
    import torch
    import w4a4_post_quantization_token_b200 as kq
    V = _rows(int(p * 10))
    M, K = V.shape
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((M, K // 32), dtype=torch.uint8, device="cuda")
    kq.debug_encode_lp_f32(torch.from_numpy(V).cuda(), p, codes, scales)
    torch.cuda.synchronize()
    c_ref, s_ref, _ = lpfit.encode_lp(V.astype(np.float64), p)
    s_gpu = scales.cpu().numpy()
    gap = lpfit.objective_gap(V.astype(np.float64), p)
    diff = s_gpu != s_ref
    assert np.all(gap[diff] < 1e-12), (np.count_nonzero(diff), gap[diff].max(initial=0))
    same = np.repeat(~diff, 32, axis=1)
    c_gpu = unpack_nibbles(codes.cpu().numpy())
    np.testing.assert_array_equal(c_gpu[same], c_ref[same])
    # the fit did move scales somewhere (the rows have heavy tails)
    from oracle import mxfp4
    _, s_ocp = mxfp4.encode(V.astype(np.float64))
    if p < 2.0:
        assert np.count_nonzero(s_gpu != s_ocp) > 0


def test_layer_with_lp_fit(cuda_device):
    import torch
    import w4a4_post_quantization_token_b200 as kq
    w = workload(2, M=300, N=768)
    inp = make_inputs(w)
    prep = olayer.prepare(inp["W"], inp["T"], w.rank, lp=1.0)
    L = make_layer(w, inp["T"])
    wbuf = torch.empty(kq.weights_bytes(L), dtype=torch.uint8, device="cuda")
    ws = torch.empty(kq.prepare_ws_bytes(L), dtype=torch.uint8, device="cuda")
    kq.prepare_weights_lp(L, 1.0, inp["W"].cuda(), wbuf, ws)
    X = inp["X"].cuda()
    act = torch.empty(kq.act_bytes(L, w.M), dtype=torch.uint8, device="cuda")
    Y = torch.empty((w.M, w.N), dtype=torch.float32, device="cuda")
    kq.linear(L, wbuf, X, Y, act)
    torch.cuda.synchronize()
    Yref = olayer.linear(inp["X"], inp["T"], w.center, prep)
    assert rel_fro(Y.cpu().double().numpy(), Yref) <= 1e-3
