"""GPU: the online half against the oracle.

* centring + block transform (kq_debug_transform): per 32-block max|d| <= 1e-5 of the
  block's max and relative Frobenius <= 1e-5 (fp32 kernel vs fp64 oracle);
* the full quantize kernel (kq_quantize_act): MXFP4 codes/scales equal to the oracle's
  except where the oracle's float32 value sits within 2e-5 of a rounding decision point,
  measured in units of its block's maximum (the unit of the transform's error bound);
  token means; low-rank input U within fp16 rounding."""
import numpy as np
import pytest

from oracle import bf16 as obf16
from oracle import layer as olayer
from oracle import mxfp4, transforms
from synthetic import make_inputs, make_transform, workload
from tests.kqtest import make_layer, pack_oracle_weights, unpack_nibbles

pytestmark = pytest.mark.gpu

CASES = [  # (workload law, overrides): ragged M, every transform, centring on/off
    (1, dict(M=200)),
    (2, dict(M=131)),
    (3, dict(M=70, N=256, rank=32)),
    (4, dict(M=67, N=256, rank=32)),
    (5, dict(M=129, N=256, rank=64)),
    (1, dict(M=33, center=False, K=64, N=64, rank=0)),
    (2, dict(M=50, center=True, K=2048, N=128, rank=5)),
    # the streaming Kronecker path: K % 64 == 32 (a half piece), centring with rank 0 (the
    # statistics alone), a low-rank branch without centring, several row tiles at S = 1
    (1, dict(M=45, K=96, N=64, rank=4)),
    (3, dict(M=140, K=160, N=64, rank=8)),
    (5, dict(M=77, N=64, rank=0)),
    (1, dict(M=260, center=False, rank=16)),
    (3, dict(M=1300, K=3072, N=64, rank=32)),
]


def _ids(c):
    return f"w{c[0]}-" + "-".join(f"{k}{v}" for k, v in c[1].items())


def _setup(index, kw):
    import torch
    w = workload(index, **kw)
    inp = make_inputs(w)
    prep = olayer.prepare(inp["W"], inp["T"], w.rank)
    L = make_layer(w, inp["T"])
    wbuf = pack_oracle_weights(L, prep)
    X = inp["X"].cuda()
    return w, inp, prep, L, wbuf, X


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_transform_matches_oracle(cuda_device, case):
    import torch
    import w4a4_post_quantization_token_b200 as kq
    w, inp, prep, L, wbuf, X = _setup(*case)
    Xt = torch.empty((w.M, w.K), dtype=torch.float32, device="cuda")
    mu = torch.empty((w.M,), dtype=torch.float32, device="cuda")
    kq.debug_transform(L, wbuf, X, Xt, mu)
    torch.cuda.synchronize()
    ref_mu, Xc = olayer.center(inp["X"].double().numpy(), w.center)
    ref = transforms.apply(Xc, inp["T"])
    got = Xt.cpu().double().numpy()
    d = np.abs(got - ref).reshape(w.M, -1, 32).max(axis=2)
    bmax = np.abs(ref).reshape(w.M, -1, 32).max(axis=2)
    assert np.all(d <= 1e-5 * np.maximum(bmax, 1e-30)), float(np.max(d / np.maximum(bmax, 1e-30)))
    assert np.linalg.norm(got - ref) <= 1e-5 * np.linalg.norm(ref)
    np.testing.assert_allclose(mu.cpu().numpy(), ref_mu, rtol=1e-6, atol=1e-6 * np.abs(ref_mu).max() + 1e-30)


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_quantize_act_matches_oracle(cuda_device, case):
    import torch
    import w4a4_post_quantization_token_b200 as kq
    w, inp, prep, L, wbuf, X = _setup(*case)
    act = torch.empty(kq.act_bytes(L, w.M), dtype=torch.uint8, device="cuda")
    kq.quantize_act(L, wbuf, X, act)
    codes = torch.empty((w.M, w.K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((w.M, w.K // 32), dtype=torch.uint8, device="cuda")
    mu = torch.empty((w.M,), dtype=torch.float32, device="cuda")
    U = torch.empty((w.M, max(w.rank, 1)), dtype=torch.float16, device="cuda")
    kq.act_unpack(L, act, w.M, codes, scales, mu, U if w.rank else None)
    assert kq.last_device_error(L, act, w.M) == 0
    ref = olayer.quantize_act(inp["X"], inp["T"], w.center, prep)

    gs = scales.cpu().numpy()
    gc = unpack_nibbles(codes.cpu().numpy())
    margin = mxfp4.decision_margin(ref["Xt32"])
    # a scale may differ only where the block max sits at a power-of-two boundary
    bad_s = gs != ref["scales"]
    blk_margin = margin.reshape(w.M, -1, 32).min(axis=2)
    assert np.all(blk_margin[bad_s] < 2e-5)
    ok_blocks = np.repeat(~bad_s, 32, axis=1)
    # +0 (0x0) and -0 (0x8) decode to the same value: where the transform cancels exactly,
    # the sign of the zero is an artefact of summation order (fp32 kernel vs fp64 oracle)
    canon = lambda c: np.where((c & 7) == 0, 0, c)
    bad_c = (canon(gc) != canon(ref["codes"])) & ok_blocks
    if not np.all(margin[bad_c] < 2e-5):
        # diagnostics: the same kernel's transform output (debug entry) at the mismatches
        Xt = torch.empty((w.M, w.K), dtype=torch.float32, device="cuda")
        mud = torch.empty((w.M,), dtype=torch.float32, device="cuda")
        kq.debug_transform(L, wbuf, X, Xt, mud)
        xt = Xt.cpu().double().numpy()
        rr, cc = np.nonzero(bad_c & (margin >= 2e-5))
        lines = []
        for r_, c_ in list(zip(rr, cc))[:12]:
            b_ = c_ // 32
            blk = ref["Xt32"][r_, 32 * b_:32 * b_ + 32]
            dc, _ = mxfp4.encode(xt[r_:r_ + 1, 32 * b_:32 * b_ + 32].astype(np.float32).astype(np.float64))
            lines.append(f"row {r_} col {c_} (blk {b_}, lane-blk {b_ % 32}) oracle v={ref['Xt32'][r_, c_]:.6g} "
                         f"gpu-debug v={xt[r_, c_]:.6g} amax={np.abs(blk).max():.4g} "
                         f"code oracle={ref['codes'][r_, c_]} gpu={gc[r_, c_]} enc(debug)={dc[0, c_ % 32]}")
        raise AssertionError(f"{bad_c.sum()} code mismatches away from a decision point:\n" +
                             "\n".join(lines))
    assert bad_c.mean() < 1e-3
    np.testing.assert_allclose(mu.cpu().numpy(), ref["mu"], rtol=1e-6,
                               atol=1e-6 * (np.abs(ref["mu"]).max() + 1.0))
    if w.rank:
        Ug = U.float().cpu().double().numpy()
        Ur = ref["U"]
        rms = np.sqrt(np.mean(Ur ** 2))
        # fp16 rounding (2^-11 relative) plus the hi/lo bf16 representation of L1'
        assert np.all(np.abs(Ug - Ur) <= 2.0 ** -10 * np.abs(Ur) + 1e-4 * rms)


def test_quantize_is_deterministic(cuda_device):
    import torch
    import w4a4_post_quantization_token_b200 as kq
    w, inp, prep, L, wbuf, X = _setup(5, dict(M=300, N=256, rank=64))
    outs = []
    for _ in range(2):
        act = torch.full((kq.act_bytes(L, w.M),), 0x5A, dtype=torch.uint8, device="cuda")
        kq.quantize_act(L, wbuf, X, act)
        torch.cuda.synchronize()
        act[:4] = 0                                  # error word
        outs.append(act.cpu().numpy())
    # the codes region is identical run to run
    np.testing.assert_array_equal(outs[0][256:256 + w.M * w.K // 2], outs[1][256:256 + w.M * w.K // 2])
