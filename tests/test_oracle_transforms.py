"""Pins for the oracle's block transforms (CPU only).

Kronecker: the explicit np.kron block against the factored A^T X_m B apply and an
element formula written out with loops; Hadamard: H H^T = 32 I, Sylvester
matrix against the fast transform; RPBH: orthogonality of the whole rotation;
fold: (X P)(P^-1 W) = X W (KroQuant section 01 identity); special cases."""
import numpy as np
import pytest

from oracle import transforms as tr
from synthetic import make_transform, workload


def _kron_T(seed=0):
    return make_transform(workload(1))


def _rpbh_T(K, seed=5):
    rng = np.random.default_rng(seed)
    return {"kind": "rpbh", "perm": rng.permutation(K).astype(np.int32),
            "sign": np.where(rng.integers(0, 2, K) == 1, 1, -1).astype(np.int8)}


def test_kron_block_element_formula():
    T = _kron_T()
    A, B = T["A"].astype(np.float64), T["B"].astype(np.float64)
    P = tr.kron_block(A, B)
    for i in range(4):
        for j in range(8):
            for k in range(4):
                for l in range(8):
                    assert P[8 * i + j, 8 * k + l] == A[i, k] * B[j, l]


def test_kron_explicit_vs_factored():
    T = _kron_T()
    rng = np.random.default_rng(1)
    X = rng.standard_normal((17, 32 * 9)) * 10
    a = tr.kron_apply_explicit(X, T["A"], T["B"])
    b = tr.kron_apply_factored(X, T["A"], T["B"])
    assert np.max(np.abs(a - b)) <= 1e-12 * np.max(np.abs(a))


def test_kron_diagonal_special_case():
    # A = diag(1,2,3,4), B = I: element 8i+j is scaled by A[i,i]
    A = np.diag([1.0, 2.0, 3.0, 4.0])
    B = np.eye(8)
    x = np.arange(64, dtype=np.float64)[None, :]
    y = tr.kron_apply_explicit(x, A, B)
    want = x * np.tile(np.repeat([1.0, 2.0, 3.0, 4.0], 8), 2)[None, :]
    np.testing.assert_array_equal(y, want)
    # A = B = I reduces to the identity (plain MXFP4 without a transform)
    np.testing.assert_array_equal(tr.kron_apply_explicit(x, np.eye(4), np.eye(8)), x)


def test_hadamard_orthogonality_and_fwht():
    H = tr.sylvester_hadamard(32)
    np.testing.assert_array_equal(H @ H.T, 32 * np.eye(32))
    np.testing.assert_array_equal(H, H.T)
    rng = np.random.default_rng(2)
    v = rng.standard_normal((5, 32))
    assert np.max(np.abs(tr.fwht(v) - v @ H)) < 1e-12
    # first row all ones, row 1 alternates sign (Sylvester order)
    np.testing.assert_array_equal(H[0], np.ones(32))
    np.testing.assert_array_equal(H[1], np.tile([1.0, -1.0], 16))


def test_rpbh_is_orthogonal():
    K = 128
    T = _rpbh_T(K)
    P = tr.dense_matrix(T, K)
    assert np.max(np.abs(P @ P.T - np.eye(K))) < 1e-13
    # RPBH(x) = x Pi H D: with identity permutation and +1 signs it is the normalised FWHT
    T0 = {"kind": "rpbh", "perm": np.arange(K, dtype=np.int32), "sign": np.ones(K, np.int8)}
    x = np.random.default_rng(0).standard_normal((3, K))
    want = tr.fwht(x.reshape(3, 4, 32)).reshape(3, K) / np.sqrt(32)
    assert np.max(np.abs(tr.apply(x, T0) - want)) < 1e-12


def test_rpbh_order_permute_then_hadamard_then_sign():
    K = 64
    T = _rpbh_T(K, seed=9)
    x = np.zeros((1, K))
    x[0, T["perm"][5]] = 1.0                 # after the gather, the 1 sits at position 5
    y = tr.apply(x, T)
    H = tr.sylvester_hadamard(32)
    want = np.zeros(K)
    want[:32] = H[5] / np.sqrt(32)           # e_5 H = row 5 of H (block 0)
    want *= T["sign"]
    np.testing.assert_allclose(y[0], want, rtol=0, atol=1e-15)


@pytest.mark.parametrize("kind", ["kron", "rpbh"])
def test_fold_identity(kind):
    K, N, M = 32 * 6, 40, 9
    T = _kron_T() if kind == "kron" else _rpbh_T(K)
    rng = np.random.default_rng(4)
    X = rng.standard_normal((M, K))
    W = rng.standard_normal((K, N))
    Y = X @ W
    Yf = tr.apply(X, T) @ tr.inverse_fold(W, T)
    assert np.linalg.norm(Yf - Y) <= 1e-12 * np.linalg.norm(Y)
    # the dense matrix agrees with the blockwise apply and with the fold
    P = tr.dense_matrix(T, K)
    assert np.max(np.abs(X @ P - tr.apply(X, T))) < 1e-12
    assert np.max(np.abs(np.linalg.inv(P) @ W - tr.inverse_fold(W, T))) < 1e-10


@pytest.mark.parametrize("kind", ["kron", "rpbh"])
def test_forward_fold_is_P_times_L(kind):
    K, r = 32 * 4, 7
    T = _kron_T() if kind == "kron" else _rpbh_T(K)
    L = np.random.default_rng(6).standard_normal((K, r))
    P = tr.dense_matrix(T, K)
    assert np.max(np.abs(P @ L - tr.forward_fold(L, T))) < 1e-12
