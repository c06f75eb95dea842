"""GPU: Lloyd-Max codebook activations with a per-token sigma (the codebook variant of the
layer) against the oracle.

* quantize: sigma within 1e-6; each value's codebook level equal to the oracle's except
  where the oracle's |Xt| / sigma lies within 2e-5 of a threshold (or, for the sign,
  within 2e-5 of zero), the decision the fp32 kernel and the fp64 oracle can take
  differently; the stored fp16 value within fp16 rounding of sigma times the level;
  token means and U as in the MXFP4 layer;
* GEMM alone: the oracle's own fp16 operand packed into the workspace, so the fp16
  tensor-core contraction of operand x decoded residual + U L2 + mu s is compared up to
  fp32 accumulation (<= 1e-5 relative);
* the whole layer and the GPU prepare: the GPU's codebook decisions are first checked
  against the oracle's (equal away from a threshold, as above); the output is then
  compared, at <= 1e-3 relative Frobenius, with the oracle's arithmetic on those
  decisions. A decision within 2e-5 of a threshold may go either way (fp32 kernel, fp64
  oracle), and one flip moves a value by a level spacing (~0.28 sigma), i.e. the output
  by about 0.28 / sqrt(M K) relative: 7e-4 for one flip in a 131 x 1152 case, so the
  plain comparison with the oracle's own decisions is only bounded loosely (<= 1e-2)."""
import numpy as np
import pytest

from oracle import layer as olayer
from oracle import lloydmax as lm
from synthetic import make_inputs, workload
from tests.kqtest import pack_oracle_weights, rel_fro

pytestmark = pytest.mark.gpu

CASES = [
    (2, dict(M=131, N=256, center=True)),                      # RPBH, r 32, centred
    (2, dict(M=300, N=512)),                                    # RPBH, not centred
    (4, dict(M=67, N=256, rank=0)),                             # RPBH K 12288, post-GELU law
    (2, dict(M=50, K=2048, N=128, rank=5, center=True, transform="none")),
    (2, dict(M=1, N=256, center=True)),
]


def _ids(c):
    return f"w{c[0]}-" + "-".join(f"{k}{v}" for k, v in c[1].items())


def _setup(index, kw):
    import w4a4_post_quantization_token_b200 as kq
    w = workload(index, **kw)
    inp = make_inputs(w)
    prep = olayer.prepare(inp["W"], inp["T"], w.rank)
    L = kq.Layer(w.K, w.N, w.rank, w.center, inp["T"], codebook="lloydmax")
    wbuf = pack_oracle_weights(L, prep)
    return w, inp, prep, L, wbuf


def _quantize(L, wbuf, w, X):
    import torch
    import w4a4_post_quantization_token_b200 as kq
    act = torch.empty(kq.act_bytes(L, w.M), dtype=torch.uint8, device="cuda")
    kq.quantize_act(L, wbuf, X.cuda(), act)
    A = torch.empty((w.M, w.K), dtype=torch.float16, device="cuda")
    sig = torch.empty(w.M, dtype=torch.float32, device="cuda")
    mu = torch.empty(w.M, dtype=torch.float32, device="cuda")
    U = torch.empty((w.M, max(w.rank, 1)), dtype=torch.float16, device="cuda")
    kq.act_unpack(L, act, w.M, A, sig, mu, U if w.rank else None)
    assert kq.last_device_error(L, act, w.M) == 0
    return (act, A.double().cpu().numpy(), sig.double().cpu().numpy(), mu.cpu().numpy(),
            U.float().cpu().double().numpy())


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_quantize_matches_oracle(cuda_device, case):
    w, inp, prep, L, wbuf = _setup(*case)
    _, A, sig, mu, U = _quantize(L, wbuf, w, inp["X"])
    ref = lm.quantize_act(inp["X"].double().numpy(), inp["T"], w.center, prep)
    np.testing.assert_allclose(sig, ref["sigma"], rtol=1e-6)
    pos, th = lm.magnitudes()
    z = np.abs(ref["Xt"]) / ref["sigma"][:, None]
    margin = np.min(np.abs(z[..., None] - th), axis=-1)
    # the GPU's level: nearest magnitude of |A| / sigma (fp16 rounding moves it by < 2^-11)
    lev_g = np.argmin(np.abs(np.abs(A)[..., None] / sig[:, None, None] - pos), axis=-1)
    lev_o = ref["codes"] & 7
    bad = lev_g != lev_o
    assert np.all(margin[bad] < 2e-5), int(np.sum(margin[bad] >= 2e-5))
    assert bad.mean() < 1e-3
    sgn_bad = np.signbit(A) != (ref["codes"] >= 8)
    assert np.all(z[sgn_bad] < 2e-5)
    want = pos[lev_g] * sig[:, None]
    assert np.all(np.abs(np.abs(A) - want) <= 2.0 ** -11 * want + 1e-30)
    np.testing.assert_allclose(mu, ref["mu"], rtol=1e-6, atol=1e-6 * (np.abs(ref["mu"]).max() + 1.0))
    if w.rank:
        rms = np.sqrt(np.mean(ref["U"] ** 2))
        assert np.all(np.abs(U[:, :w.rank] - ref["U"]) <= 2.0 ** -10 * np.abs(ref["U"]) + 1e-4 * rms)


@pytest.mark.parametrize("case", CASES[:4], ids=_ids)
def test_gemm_on_the_oracle_operand(cuda_device, case):
    import torch
    import w4a4_post_quantization_token_b200 as kq
    w, inp, prep, L, wbuf = _setup(*case)
    ref = lm.quantize_act(inp["X"].double().numpy(), inp["T"], w.center, prep)
    act = torch.empty(kq.act_bytes(L, w.M), dtype=torch.uint8, device="cuda")
    A16 = torch.from_numpy(ref["A16"].astype(np.float16)).cuda()
    sig = torch.from_numpy(ref["sigma"].astype(np.float32)).cuda()
    mu = torch.from_numpy(ref["mu"].astype(np.float32)).cuda()
    U = torch.from_numpy(ref["U"].astype(np.float16)).cuda() if w.rank else None
    kq.act_pack(L, A16, sig, mu, U, w.M, act)
    Y = torch.empty((w.M, w.N), dtype=torch.float32, device="cuda")
    kq.gemm(L, wbuf, act, w.M, Y)
    torch.cuda.synchronize()
    Uq = ref["U"].astype(np.float16).astype(np.float64) if w.rank else 0.0
    mu32 = ref["mu"].astype(np.float32).astype(np.float64)
    s32 = prep["s"].astype(np.float32).astype(np.float64)
    L2 = prep["L2"].astype(np.float16).astype(np.float64) if w.rank else 0.0
    Yref = ref["A16"] @ lm.residual_fp16(prep) + (Uq @ L2 if w.rank else 0.0) + np.outer(mu32, s32)
    assert rel_fro(Y.cpu().double().numpy(), Yref) <= 1e-5


def _linear(L, wbuf, X, N):
    """Y [M, N] float64, plus the workspace's fp16 operand and sigma."""
    import torch
    import w4a4_post_quantization_token_b200 as kq
    M = X.shape[0]
    act = torch.empty(kq.act_bytes(L, M), dtype=torch.uint8, device="cuda")
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    kq.linear(L, wbuf, X.cuda(), Y, act)
    A = torch.empty((M, L.K), dtype=torch.float16, device="cuda")
    sig = torch.empty(M, dtype=torch.float32, device="cuda")
    kq.act_unpack(L, act, M, A, sig)
    torch.cuda.synchronize()
    assert kq.last_device_error(L, act, M) == 0
    return Y.cpu().double().numpy(), A.double().cpu().numpy(), sig.double().cpu().numpy()


def _check_layer(w, inp, prep, Y, A, sig, tol=1e-3):
    ref = lm.quantize_act(inp["X"].double().numpy(), inp["T"], w.center, prep)
    pos, th = lm.magnitudes()
    z = np.abs(ref["Xt"]) / ref["sigma"][:, None]
    margin = np.min(np.abs(z[..., None] - th), axis=-1)
    lev_g = np.argmin(np.abs(np.abs(A)[..., None] / sig[:, None, None] - pos), axis=-1)
    codes_g = ((np.signbit(A).astype(np.int64) << 3) | lev_g).astype(np.uint8)
    bad = codes_g != ref["codes"]
    near = np.where(codes_g & 7 != ref["codes"] & 7, margin, z)
    assert np.all(near[bad] < 2e-5), int(np.sum(near[bad] >= 2e-5))
    # the oracle's arithmetic on the GPU's (validated) decisions
    Yg_ref = (lm.fp16_operand(codes_g, ref["sigma"]) @ lm.residual_fp16(prep) + ref["U"] @ prep["L2"]
              + np.outer(ref["mu"], prep["s"]))
    err = rel_fro(Y, Yg_ref)
    assert err <= tol, (err, int(bad.sum()))
    Yref = lm.linear(inp["X"].double().numpy(), inp["T"], w.center, prep)
    assert rel_fro(Y, Yref) <= 1e-2


@pytest.mark.parametrize("case", CASES + [(2, dict(M=127, N=256, center=True)),
                                          (2, dict(M=129, N=192))], ids=_ids)
def test_layer_matches_oracle(cuda_device, case):
    w, inp, prep, L, wbuf = _setup(*case)
    _check_layer(w, inp, prep, *_linear(L, wbuf, inp["X"], w.N))


def test_prepare_on_gpu(cuda_device):
    """kq_prepare_weights decodes the residual to fp16 for the codebook layer itself."""
    import torch
    import w4a4_post_quantization_token_b200 as kq
    w, inp, prep, L, _ = _setup(2, dict(M=260, N=512, center=True))
    wbuf = torch.empty(kq.weights_bytes(L), dtype=torch.uint8, device="cuda")
    ws = torch.empty(kq.prepare_ws_bytes(L), dtype=torch.uint8, device="cuda")
    kq.prepare_weights(L, inp["W"].cuda(), wbuf, ws)
    # the GPU's own SVD and residual encode differ from the oracle's at rounding level
    # (their parity is tested with the MXFP4 layer); that adds to the bound here
    _check_layer(w, inp, prep, *_linear(L, wbuf, inp["X"], w.N), tol=2e-3)


@pytest.mark.parametrize("index", [2, 4])
def test_layer_full_size_sampled(cuda_device, index):
    """The full RPBH workloads in the bench's launch configuration; the oracle checks 48
    sampled rows (incl. the last ones) on the GPU's validated decisions."""
    import w4a4_post_quantization_token_b200 as kq
    from tests.kqtest import cached
    w, inp, prep = cached(index)
    L = kq.Layer(w.K, w.N, w.rank, w.center, inp["T"], codebook="lloydmax")
    wbuf = pack_oracle_weights(L, prep)
    Y, A, sig = _linear(L, wbuf, inp["X"], w.N)
    rng = np.random.default_rng(index)
    rows = np.unique(np.concatenate([rng.choice(w.M, 40, replace=False),
                                     np.arange(max(0, w.M - 8), w.M)]))
    sub = {"X": inp["X"][rows], "T": inp["T"]}
    _check_layer(workload(index, M=len(rows)), sub, prep, Y[rows], A[rows], sig[rows])
