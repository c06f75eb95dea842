"""Pins for the oracle's layer composition (CPU only).

Centring and exact mean restore (CentriQ abstract), the SVD split
(Eckart-Young; SVDQuant section 3), the L1' = P L1 rewrite, bf16 rounding, and
an end-to-end special case whose quantization is lossless so that the whole
composition must reproduce X W exactly (catches transposed operands, dropped
terms and wrong signs)."""
import numpy as np
import pytest

from oracle import bf16, layer, mxfp4, transforms as tr
from synthetic import exact_grid_inputs, make_inputs, workload


def test_bf16_rounding_against_bit_truncation():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(20000) * np.exp2(rng.integers(-30, 30, 20000))
    r = bf16.round_bf16(x)
    # r is a bf16 value, and no bf16 value is nearer (checked with the two neighbours)
    f = r.astype(np.float32)
    assert np.all((f.view(np.uint32) & 0xFFFF) == 0)
    up = (f.view(np.uint32) + 0x10000).view(np.float32).astype(np.float64)
    dn = (f.view(np.uint32) - 0x10000).view(np.float32).astype(np.float64)
    assert np.all(np.abs(x - r) <= np.abs(x - up))
    assert np.all(np.abs(x - r) <= np.abs(x - dn))
    # ties go to an even last bit
    tie = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8)])
    np.testing.assert_array_equal(bf16.round_bf16(tie), [1.0, 1.0 + 4 * 2 ** -8, -1.0])


def test_centering_rows_sum_to_zero_and_restore():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((11, 96)) * 3 + rng.standard_normal((11, 1)) * 5
    W = rng.standard_normal((96, 13))
    mu, Xc = layer.center(X, True)
    assert np.max(np.abs(Xc.sum(axis=1))) <= 1e-12 * 96 * np.max(np.abs(X))
    s = W.sum(axis=0)
    assert np.linalg.norm(Xc @ W + np.outer(mu, s) - X @ W) <= 1e-12 * np.linalg.norm(X @ W)
    mu0, Xc0 = layer.center(X, False)
    assert np.all(mu0 == 0) and np.array_equal(Xc0, X)


def test_eckart_young_and_rank_limits():
    rng = np.random.default_rng(2)
    W = rng.standard_normal((96, 64))
    for r in (0, 5, 64):
        if r:
            L1, L2, S = layer.truncated_svd_factors(W, r)
            resid = np.linalg.norm(W - L1 @ L2) ** 2
            assert abs(resid - np.sum(S[r:] ** 2)) <= 1e-9 * np.sum(S ** 2)
    T = {"kind": "none"}
    p0 = layer.prepare(W, T, 0)
    np.testing.assert_array_equal(p0["R"], W)          # r = 0: plain W4A4 residual
    pf = layer.prepare(W, T, 64)
    # full rank: residual is only the bf16 rounding of the factors
    assert np.linalg.norm(pf["R"]) < 1e-2 * np.linalg.norm(W)


@pytest.mark.parametrize("kind", ["kron", "rpbh"])
def test_lowrank_input_rewrite(kind):
    w = workload(1 if kind == "kron" else 2, M=20, K=128, N=48, rank=6)
    inp = make_inputs(w)
    prep = layer.prepare(inp["W"], inp["T"], w.rank)
    X = inp["X"].double().numpy()
    act = layer.quantize_act(X, inp["T"], True, prep)
    U_direct = act["Xt"] @ prep["L1"]
    U_raw = X @ prep["L1p"] - np.outer(act["mu"], prep["c1"])
    assert np.max(np.abs(U_direct - U_raw)) <= 1e-10 * np.max(np.abs(U_direct))
    np.testing.assert_allclose(prep["c1"], prep["L1p"].sum(axis=0), rtol=0, atol=0)
    # L2 and L1 are bf16 values
    for a in (prep["L1"], prep["L2"]):
        f = a.astype(np.float32)
        assert np.all(f.astype(np.float64) == a) and np.all((f.view(np.uint32) & 0xFFFF) == 0)


def test_lossless_special_case_reproduces_XW():
    """No transform, no centring, r = 0, inputs on the MXFP4 grid: every step but the
    contraction is exact, so Y_ref must equal X W exactly."""
    M, K, N = 24, 32 * 5, 40
    Xq, Wq_nk = exact_grid_inputs(M, K, N, seed=3)
    W = Wq_nk.T.astype(np.float64)                     # [K, N]
    T = {"kind": "none"}
    prep = layer.prepare(W, T, 0)
    Y = layer.linear(Xq.astype(np.float64), T, False, prep)
    np.testing.assert_array_equal(Y, Xq.astype(np.float64) @ W)


def test_centering_restores_mean_exactly_on_grid():
    """Centring with a per-token shift chosen so that X_c is on the grid: the rank-1
    branch must restore the shift exactly (CentriQ: exact mean restore)."""
    M, K, N = 16, 64, 24
    Xq, Wq_nk = exact_grid_inputs(M, K, N, seed=4)
    Xq = Xq.astype(np.float64)
    Xc = Xq - Xq.mean(axis=1, keepdims=True)
    shift = np.arange(M, dtype=np.float64)[:, None] * 0.5
    W = Wq_nk.T.astype(np.float64)
    T = {"kind": "none"}
    prep = layer.prepare(W, T, 0)
    act = layer.quantize_act(Xc + shift, T, True, prep)
    assert np.max(np.abs(act["mu"] - shift[:, 0])) < 1e-12
    Y = layer.linear_from_parts(act, prep)
    Yq = mxfp4.decode(*mxfp4.encode(bf16.round_f32(Xc))) @ W
    assert np.max(np.abs(Y - (Yq + shift * W.sum(axis=0)[None, :]))) < 1e-9


def test_layer_error_small_and_rotation_helps():
    """The oracle layer approximates X W; on outlier-heavy inputs the permuted
    block-Hadamard rotation lowers the error against no transform (OrbitQuant
    section 03). Loose sanity bound, not a pin. (The synthetic Kronecker factors
    are near the identity, not learned, so no such claim is made for them.)"""
    w = workload(2, M=64, K=256, N=96, rank=8)
    inp = make_inputs(w)
    X = inp["X"].double().numpy()
    W = inp["W"].double().numpy()
    Y = X @ W
    prep = layer.prepare(W, inp["T"], w.rank)
    err_t = np.linalg.norm(layer.linear(X, inp["T"], False, prep) - Y) / np.linalg.norm(Y)
    prep0 = layer.prepare(W, {"kind": "none"}, w.rank)
    err_0 = np.linalg.norm(layer.linear(X, {"kind": "none"}, False, prep0) - Y) / np.linalg.norm(Y)
    assert err_t < 0.25
    assert err_t < err_0


def test_centering_helps_with_token_shift():
    """With a large per-token shift, centring before the transform lowers the
    error (CentriQ abstract: the per-token mean otherwise sets the range)."""
    w = workload(5, M=64, K=3072, N=96, rank=8)
    inp = make_inputs(w)
    X = inp["X"].double().numpy()
    W = inp["W"].double().numpy()
    Y = X @ W
    prep = layer.prepare(W, inp["T"], w.rank)
    err_c = np.linalg.norm(layer.linear(X, inp["T"], True, prep) - Y) / np.linalg.norm(Y)
    err_n = np.linalg.norm(layer.linear(X, inp["T"], False, prep) - Y) / np.linalg.norm(Y)
    assert err_c < err_n


@pytest.mark.parametrize("law,kind", [(1, "kron"), (2, "rpbh")])
def test_exact_rank_weight_is_carried_by_the_lowrank_branch(law, kind):
    """A weight of exact rank r, W = B1 B2, with rank r kept (SVDQuant section 3): the
    transform-folded weight W' = P^{-1} W has rank r too, so the 16-bit factors hold all
    of it and the 4-bit residual R = W' - L1 L2 holds only their bf16 rounding (about
    2^-8 of W'). The layer output is then X W up to the MXFP4 error of the small product
    Xt R: Y - X W = deq(Q(Xt)) deq(Q(R)) - Xt R, well under 1e-2 of X W. The pin is the
    identity Xt L1 L2 + Xt R + mu s = X W (centring restores mu s exactly, the transform
    cancels against its fold): dropping the U L2 term, forming U from the centred input
    before the transform instead of Xt, or losing mu s each move Y by O(1) of X W, which
    the test checks on the same data."""
    M, K, N, r = 24, 64, 40, 4
    rng = np.random.default_rng(11)
    B1 = rng.integers(-3, 4, size=(K, r)).astype(np.float64) * 2.0 ** -3
    B2 = rng.integers(-3, 4, size=(r, N)).astype(np.float64) * 2.0 ** -4
    W = B1 @ B2
    assert np.linalg.matrix_rank(W) == r
    w = workload(law, M=M, K=K, N=N, rank=r, transform=kind, center=True)
    inp = make_inputs(w)
    X = inp["X"].double().numpy()
    T = inp["T"]
    prep = layer.prepare(W, T, r)
    # the residual is only the rounding of the factors
    assert np.linalg.norm(prep["R"]) < 2.0 ** -7 * np.linalg.norm(prep["Wp"])
    act = layer.quantize_act(X, T, True, prep)
    Y = layer.linear_from_parts(act, prep)
    XW = X @ W
    nrm = np.linalg.norm(XW)
    err = np.linalg.norm(Y - XW) / nrm
    assert err < 1e-2, err
    # each plausible slip moves the output by O(1)
    Xq = mxfp4.decode(act["codes"], act["scales"])
    Rq = mxfp4.decode(prep["r_codes"], prep["r_scales"]).T
    no_lowrank = Xq @ Rq + np.outer(act["mu"], prep["s"])
    u_before_transform = Xq @ Rq + (act["Xc"] @ prep["L1"]) @ prep["L2"] + np.outer(act["mu"], prep["s"])
    no_restore = Xq @ Rq + act["U"] @ prep["L2"]
    for wrong in (no_lowrank, no_restore):
        assert np.linalg.norm(wrong - XW) / nrm > 0.2
    # the transform is close to the identity for the Kronecker law (I + N(0, 0.1)
    # factors), so forming U before it is a smaller, still clearly visible slip
    assert np.linalg.norm(u_before_transform - XW) / nrm > 10 * err
