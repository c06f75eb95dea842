"""GPU: the fused LayerNorm front-end against the oracle.

The reference result is the oracle's layer applied to the oracle's LayerNorm of the bf16
tokens (float64 throughout): y = LayerNorm(x), then centring, block transform, MXFP4,
low-rank branch and mean restore on y. The kernel normalises in fp32 with fp64 row
statistics, so the bars are those of the plain layer: the transform output within 1e-5
of each block's maximum, codes and scales equal except next to a rounding decision
point, the token means of y within 1e-6, U within fp16 rounding, and the whole layer
within 1e-3 relative Frobenius error. Cases span several 128-row tiles with ragged M,
every transform kind, ranks 0 to 64, and the full offline preparation on the GPU."""
import numpy as np
import pytest

from oracle import layer as olayer
from oracle import layernorm as oln
from oracle import mxfp4, transforms
from synthetic import make_inputs, make_layernorm, workload
from tests.kqtest import pack_oracle_weights, rel_fro, unpack_nibbles

pytestmark = pytest.mark.gpu

CASES = [
    (1, dict(M=200)),                                               # Kronecker, r 16
    (2, dict(M=131, N=256, center=True)),                           # RPBH, r 32
    (3, dict(M=70, N=256, rank=64)),                                # Kronecker, r 64
    (4, dict(M=67, N=256, center=True, rank=0)),                    # RPBH, K 12288, no branch
    (2, dict(M=50, K=2048, N=128, rank=5, center=True, transform="none")),
]


def _ids(c):
    return f"w{c[0]}-" + "-".join(f"{k}{v}" for k, v in c[1].items())


def _setup(index, kw):
    import torch
    import w4a4_post_quantization_token_b200 as kq
    w = workload(index, **kw)
    inp = make_inputs(w)
    ln = make_layernorm(w)
    Y = oln.layernorm(inp["X"].double().numpy(), ln["gamma"], ln["beta"], ln["eps"])
    prep = olayer.prepare(inp["W"], inp["T"], w.rank)
    L = kq.Layer(w.K, w.N, w.rank, True, inp["T"], layernorm=ln)
    wbuf = pack_oracle_weights(L, prep)
    return w, inp, ln, Y, prep, L, wbuf, inp["X"].cuda()


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_transform_matches_oracle(cuda_device, case):
    import torch
    import w4a4_post_quantization_token_b200 as kq
    w, inp, ln, Y, prep, L, wbuf, X = _setup(*case)
    Xt = torch.empty((w.M, w.K), dtype=torch.float32, device="cuda")
    mu = torch.empty((w.M,), dtype=torch.float32, device="cuda")
    kq.debug_transform(L, wbuf, X, Xt, mu)
    torch.cuda.synchronize()
    ref_mu, Yc = olayer.center(Y, True)
    ref = transforms.apply(Yc, inp["T"])
    got = Xt.cpu().double().numpy()
    d = np.abs(got - ref).reshape(w.M, -1, 32).max(axis=2)
    bmax = np.abs(ref).reshape(w.M, -1, 32).max(axis=2)
    assert np.all(d <= 1e-5 * np.maximum(bmax, 1e-30)), float(np.max(d / np.maximum(bmax, 1e-30)))
    assert np.linalg.norm(got - ref) <= 1e-5 * np.linalg.norm(ref)
    np.testing.assert_allclose(mu.cpu().numpy(), ref_mu, rtol=1e-6,
                               atol=1e-6 * (np.abs(ref_mu).max() + 1.0))


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_quantize_act_matches_oracle(cuda_device, case):
    import torch
    import w4a4_post_quantization_token_b200 as kq
    w, inp, ln, Y, prep, L, wbuf, X = _setup(*case)
    act = torch.empty(kq.act_bytes(L, w.M), dtype=torch.uint8, device="cuda")
    kq.quantize_act(L, wbuf, X, act)
    codes = torch.empty((w.M, w.K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((w.M, w.K // 32), dtype=torch.uint8, device="cuda")
    mu = torch.empty((w.M,), dtype=torch.float32, device="cuda")
    U = torch.empty((w.M, max(w.rank, 1)), dtype=torch.float16, device="cuda")
    kq.act_unpack(L, act, w.M, codes, scales, mu, U if w.rank else None)
    assert kq.last_device_error(L, act, w.M) == 0
    ref = olayer.quantize_act(Y, inp["T"], True, prep)

    gs = scales.cpu().numpy()
    gc = unpack_nibbles(codes.cpu().numpy())
    margin = mxfp4.decision_margin(ref["Xt32"])
    bad_s = gs != ref["scales"]
    assert np.all(margin.reshape(w.M, -1, 32).min(axis=2)[bad_s] < 2e-5)
    ok_blocks = np.repeat(~bad_s, 32, axis=1)
    canon = lambda c: np.where((c & 7) == 0, 0, c)       # +0 and -0 decode alike
    bad_c = (canon(gc) != canon(ref["codes"])) & ok_blocks
    assert np.all(margin[bad_c] < 2e-5), int(np.sum(margin[bad_c] >= 2e-5))
    assert bad_c.mean() < 1e-3
    np.testing.assert_allclose(mu.cpu().numpy(), ref["mu"], rtol=1e-6,
                               atol=1e-6 * (np.abs(ref["mu"]).max() + 1.0))
    if w.rank:
        Ug = U.float().cpu().double().numpy()
        Ur = ref["U"]
        rms = np.sqrt(np.mean(Ur ** 2))
        assert np.all(np.abs(Ug - Ur) <= 2.0 ** -10 * np.abs(Ur) + 1e-4 * rms), \
            float(np.max(np.abs(Ug - Ur) / (np.abs(Ur) + rms)))


def _run_linear(L, wbuf, X, N):
    import torch
    import w4a4_post_quantization_token_b200 as kq
    M = X.shape[0]
    act = torch.empty(kq.act_bytes(L, M), dtype=torch.uint8, device="cuda")
    Yg = torch.empty((M, N), dtype=torch.float32, device="cuda")
    kq.linear(L, wbuf, X, Yg, act)
    torch.cuda.synchronize()
    assert kq.last_device_error(L, act, M) == 0
    return Yg.cpu().double().numpy()


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_layer_matches_oracle(cuda_device, case):
    w, inp, ln, Y, prep, L, wbuf, X = _setup(*case)
    Yref = olayer.linear(Y, inp["T"], True, prep)
    err = rel_fro(_run_linear(L, wbuf, X, w.N), Yref)
    assert err <= 1e-3, err


def test_prepare_on_gpu_with_front_end(cuda_device):
    """kq_prepare_weights writes the front-end parts itself (gamma, beta, the kernel's
    table, diag(gamma) L1' and its sums); the layer then matches the oracle's."""
    import torch
    import w4a4_post_quantization_token_b200 as kq
    w, inp, ln, Y, prep, L, _, X = _setup(3, dict(M=300, N=512))
    wbuf = torch.empty(kq.weights_bytes(L), dtype=torch.uint8, device="cuda")
    ws = torch.empty(kq.prepare_ws_bytes(L), dtype=torch.uint8, device="cuda")
    kq.prepare_weights(L, inp["W"].cuda(), wbuf, ws)
    Yref = olayer.linear(Y, inp["T"], True, prep)
    assert rel_fro(_run_linear(L, wbuf, X, w.N), Yref) <= 1e-3


def test_front_end_is_not_the_plain_layer(cuda_device):
    """With gamma = 1 and beta = 0 the front-end reduces to a per-token standardisation,
    so the layer's output is the plain layer's output on standardised tokens; and
    switching the front-end on changes the result (the path is not skipped)."""
    import torch
    import w4a4_post_quantization_token_b200 as kq
    w = workload(1, M=130)
    inp = make_inputs(w)
    prep = olayer.prepare(inp["W"], inp["T"], w.rank)
    unit = {"gamma": np.ones(w.K, np.float32), "beta": np.zeros(w.K, np.float32), "eps": 1e-6}
    L = kq.Layer(w.K, w.N, w.rank, True, inp["T"], layernorm=unit)
    wbuf = pack_oracle_weights(L, prep)
    Yg = _run_linear(L, wbuf, inp["X"].cuda(), w.N)
    Xd = inp["X"].double().numpy()
    m, rstd = oln.stats(Xd, 1e-6)
    Yref = olayer.linear((Xd - m[:, None]) * rstd[:, None], inp["T"], True, prep)
    assert rel_fro(Yg, Yref) <= 1e-3
    Lp = kq.Layer(w.K, w.N, w.rank, True, inp["T"])
    plain = _run_linear(Lp, pack_oracle_weights(Lp, prep), inp["X"].cuda(), w.N)
    assert rel_fro(Yg, plain) > 0.1


@pytest.mark.parametrize("index", [2, 3, 5])
def test_layer_full_size_sampled(cuda_device, index):
    """Full workloads (centring on) with the front-end, in the bench's launch
    configuration; the oracle checks 48 sampled rows (incl. the last ones)."""
    import w4a4_post_quantization_token_b200 as kq
    from tests.kqtest import cached
    w, inp, prep = cached(index)
    ln = make_layernorm(w)
    L = kq.Layer(w.K, w.N, w.rank, True, inp["T"], layernorm=ln)
    wbuf = pack_oracle_weights(L, prep)
    Yg = _run_linear(L, wbuf, inp["X"].cuda(), w.N)
    rng = np.random.default_rng(index)
    rows = np.unique(np.concatenate([rng.choice(w.M, 40, replace=False),
                                     np.arange(max(0, w.M - 8), w.M)]))
    Y = oln.layernorm(inp["X"][rows].double().numpy(), ln["gamma"], ln["beta"], ln["eps"])
    assert rel_fro(Yg[rows], olayer.linear(Y, inp["T"], True, prep)) <= 1e-3
