"""GPU: the whole layer (kq_linear) and the offline preparation (kq_prepare_weights)
against the oracle.

Tolerance: relative Frobenius error <= 1e-3 of the oracle's fp64 dequantized product
for float32 output (the acceptance bound of the layer), <= 4e-3 for bf16 output (bf16
rounding alone is 2^-9 per element). Reduced-size cases span several 128 x 256 tiles
and ragged M; full-size cases run the bench's launch configuration on the GPU and
compare sampled rows, which the oracle computes one by one."""
import numpy as np
import pytest

from oracle import layer as olayer
from oracle import mxfp4
from synthetic import make_inputs, workload
from tests.kqtest import cached, make_layer, pack_oracle_weights, rel_fro, unpack_nibbles

pytestmark = pytest.mark.gpu

REDUCED = [
    (1, dict()),                                    # full tiny workload: 256 x 1152 -> 1152
    (2, dict(M=515, N=1024)),
    (3, dict(M=300, N=768)),
    (4, dict(M=260, N=512)),
    (5, dict(M=389, N=512)),
]


def _ids(c):
    return f"w{c[0]}-" + "-".join(f"{k}{v}" for k, v in c[1].items())


def _run_linear(L, wbuf, X, out_bf16=False):
    import torch
    import w4a4_post_quantization_token_b200 as kq
    M = X.shape[0]
    act = torch.empty(kq.act_bytes(L, M), dtype=torch.uint8, device="cuda")
    Y = torch.empty((M, L.N), dtype=torch.bfloat16 if out_bf16 else torch.float32, device="cuda")
    kq.linear(L, wbuf, X, Y, act, kq.OUT_BF16 if out_bf16 else kq.OUT_F32)
    torch.cuda.synchronize()
    assert kq.last_device_error(L, act, M) == 0
    return Y.float().cpu().double().numpy()


@pytest.mark.parametrize("case", REDUCED, ids=_ids)
def test_layer_parity_reduced(cuda_device, case):
    w, inp, prep = cached(case[0], **case[1])
    L = make_layer(w, inp["T"])
    wbuf = pack_oracle_weights(L, prep)
    X = inp["X"].cuda()
    Yref = olayer.linear(inp["X"], inp["T"], w.center, prep)
    err = rel_fro(_run_linear(L, wbuf, X), Yref)
    assert err <= 1e-3, err
    err16 = rel_fro(_run_linear(L, wbuf, X, out_bf16=True), Yref)
    assert err16 <= 4e-3, err16


@pytest.mark.parametrize("M", [1, 127, 129])
def test_layer_edge_M(cuda_device, M):
    w, inp, prep = cached(3, M=M, N=256)
    L = make_layer(w, inp["T"])
    wbuf = pack_oracle_weights(L, prep)
    Yref = olayer.linear(inp["X"], inp["T"], w.center, prep)
    assert rel_fro(_run_linear(L, wbuf, inp["X"].cuda()), Yref) <= 1e-3


@pytest.mark.parametrize("index", [1, 2, 3, 4, 5])
def test_layer_parity_full_size_sampled(cuda_device, index):
    """Full workload on the GPU; the oracle checks 48 sampled rows (incl. the last ones)."""
    w, inp, prep = cached(index)
    L = make_layer(w, inp["T"])
    wbuf = pack_oracle_weights(L, prep)
    Y = _run_linear(L, wbuf, inp["X"].cuda())
    rng = np.random.default_rng(index)
    rows = np.unique(np.concatenate([rng.choice(w.M, 40, replace=False),
                                     np.arange(max(0, w.M - 8), w.M)]))
    Xs = inp["X"][rows]
    Yref = olayer.linear(Xs, inp["T"], w.center, prep)
    assert rel_fro(Y[rows], Yref) <= 1e-3


@pytest.mark.parametrize("case", [(1, dict(N=768)), (2, dict(M=64, N=512)),
                                  (5, dict(M=64, K=1024, N=512, rank=64)),
                                  (3, dict(M=64, K=1024, N=2048, rank=7))], ids=_ids)
def test_prepare_parity(cuda_device, case):
    """kq_prepare_weights (fp64 on the GPU, eigen-decomposition of the Gram matrix) against
    the oracle's numpy SVD path: column sums, the low-rank product, residual codes
    (equal except at decision boundaries), and the layer output."""
    import torch
    import w4a4_post_quantization_token_b200 as kq
    w, inp, prep = cached(case[0], **case[1])
    L = make_layer(w, inp["T"])
    W = inp["W"].cuda()
    wbuf = torch.empty(kq.weights_bytes(L), dtype=torch.uint8, device="cuda")
    ws = torch.empty(kq.prepare_ws_bytes(L), dtype=torch.uint8, device="cuda")
    kq.prepare_weights(L, W, wbuf, ws)
    K, N, r = w.K, w.N, w.rank
    rc = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
    rs = torch.empty((N, K // 32), dtype=torch.uint8, device="cuda")
    L1p = torch.empty((K, r), dtype=torch.float32, device="cuda")
    L2 = torch.empty((r, N), dtype=torch.bfloat16, device="cuda")
    c1 = torch.empty((r,), dtype=torch.float32, device="cuda")
    s = torch.empty((N,), dtype=torch.float32, device="cuda")
    kq.weights_unpack(L, wbuf, rc, rs, L1p, L2, c1, s)
    torch.cuda.synchronize()
    np.testing.assert_allclose(s.cpu().numpy(), prep["s"], rtol=2e-7, atol=1e-7 * np.abs(prep["s"]).max())
    P_g = L1p.cpu().double().numpy() @ L2.float().cpu().double().numpy()
    P_o = prep["L1p"] @ prep["L2"]
    assert rel_fro(P_g, P_o) <= 1e-4
    # singular vectors carry a free sign per component: compare |c1|, and c1 against
    # the column sums of the stored L1'
    c1g = c1.cpu().double().numpy()
    np.testing.assert_allclose(np.abs(c1g), np.abs(prep["c1"]), rtol=1e-4,
                               atol=1e-5 * np.abs(prep["c1"]).max())
    np.testing.assert_allclose(c1g, L1p.cpu().double().numpy().sum(axis=0), rtol=1e-5,
                               atol=1e-6 * np.abs(c1g).max())
    gs = rs.cpu().numpy()
    gc = unpack_nibbles(rc.cpu().numpy())
    margin = mxfp4.decision_margin(prep["R32"].T)
    bad = (gc != prep["r_codes"]) | np.repeat(gs != prep["r_scales"], 32, axis=1)
    assert bad.mean() < 1e-3
    assert np.all(margin[bad] < 1e-4)
    Yref = olayer.linear(inp["X"], inp["T"], w.center, prep)
    assert rel_fro(_run_linear(L, wbuf, inp["X"].cuda()), Yref) <= 1e-3


def test_linear_host_buffers(cuda_device):
    import torch
    import w4a4_post_quantization_token_b200 as kq
    w, inp, prep = cached(2, M=300, N=512)
    L = make_layer(w, inp["T"])
    wbuf = pack_oracle_weights(L, prep)
    Xh = inp["X"].pin_memory()
    Yh = torch.empty((w.M, w.N), dtype=torch.float32).pin_memory()
    Xd = torch.empty_like(Xh, device="cuda")
    Yd = torch.empty((w.M, w.N), dtype=torch.float32, device="cuda")
    act = torch.empty(kq.act_bytes(L, w.M), dtype=torch.uint8, device="cuda")
    kq.linear_host(L, wbuf, Xh, Xd, Yh, Yd, act)
    torch.cuda.synchronize()
    Yref = olayer.linear(inp["X"], inp["T"], w.center, prep)
    assert rel_fro(Yh.double().numpy(), Yref) <= 1e-3


def test_linear_host_buffers_chunked(cuda_device):
    """M >= 1024 goes through the chunked host pipeline (5 chunks of 640 rows, the last one
    ragged): the device-buffer call's result up to the low-rank split, and the oracle's."""
    import torch
    import w4a4_post_quantization_token_b200 as kq
    w, inp, prep = cached(2, M=2600, N=512)
    L = make_layer(w, inp["T"])
    wbuf = pack_oracle_weights(L, prep)
    Xh = inp["X"].pin_memory()
    Yh = torch.full((w.M, w.N), float("nan"), dtype=torch.float32).pin_memory()
    Xd = torch.empty_like(Xh, device="cuda")
    Yd = torch.empty((w.M, w.N), dtype=torch.float32, device="cuda")
    act = torch.empty(kq.act_bytes(L, w.M), dtype=torch.uint8, device="cuda")
    for _ in range(2):                               # the second call reuses the pipeline
        kq.linear_host(L, wbuf, Xh, Xd, Yh, Yd, act)
    torch.cuda.synchronize()
    assert kq.last_device_error(L, act, w.M) == 0
    Ydev = torch.empty((w.M, w.N), dtype=torch.float32, device="cuda")
    kq.linear(L, wbuf, inp["X"].cuda(), Ydev, act)
    torch.cuda.synchronize()
    got = Yh.double().numpy()
    assert np.all(np.isfinite(got))
    # per-row arithmetic is the same, except that the low-rank kernel splits K by the
    # number of rows it gets, so U's fp32 partial sums (and an occasional fp16 rounding of
    # U) differ between a 640-row chunk and the 2600-row call
    assert rel_fro(got, Ydev.cpu().double().numpy()) <= 2e-5
    assert rel_fro(got, olayer.linear(inp["X"], inp["T"], w.center, prep)) <= 1e-3
