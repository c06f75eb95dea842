"""Block transforms applied to activations before quantization (oracle, test infrastructure).

Row-vector convention throughout: an activation row x (1 x K) becomes x P.

KroQuant (commentary page, section 02): the K channels are split into blocks
of 32 and every block is multiplied by the same learned invertible
P = A (x) B. With A 4x4 and B 8x8, element e = 8 i + j of a block has
(A (x) B)[(i,j),(k,l)] = A[i,k] B[j,l], so x (A (x) B) = vec_rowmajor(A^T X_m B)
with X_m[i, j] = x[8 i + j]. ``kron_apply_explicit`` forms the 32x32 matrix;
``kron_apply_factored`` uses the two small products (the pins check that they agree).

OrbitQuant (commentary page, section 03, equation RPBH(X) = X P H D):
a permutation P, a block Hadamard H and a random sign matrix D, applied in that
order. Readings: the permutation is one global permutation of the K channels,
given as a gather ``(x P)[j] = x[perm[j]]``; H is block-diagonal with Sylvester
blocks of size 32 normalised by 1/sqrt(32) so that the whole rotation is
orthogonal (the page requires an orthogonal R); D = diag(sign), sign in {+1, -1}.
"""
import numpy as np

BLOCK = 32


def sylvester_hadamard(n: int) -> np.ndarray:
    """Unnormalised Sylvester Hadamard matrix, H[i, j] = (-1)^popcount(i & j)."""
    if n & (n - 1):
        raise ValueError("n must be a power of two")
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    pc = np.vectorize(lambda v: bin(int(v)).count("1"))(i & j)
    return np.where(pc % 2 == 0, 1.0, -1.0)


def kron_block(A, B) -> np.ndarray:
    """The explicit 32x32 block matrix A (x) B (textbook Kronecker product)."""
    return np.kron(np.asarray(A, dtype=np.float64), np.asarray(B, dtype=np.float64))


def kron_apply_explicit(X, A, B) -> np.ndarray:
    """X [M, K] -> X blockdiag(A (x) B), each 32-block times the explicit 32x32 matrix."""
    X = np.asarray(X, dtype=np.float64)
    M, K = X.shape
    P = kron_block(A, B)
    return (X.reshape(M, K // BLOCK, BLOCK) @ P).reshape(M, K)


def kron_apply_factored(X, A, B) -> np.ndarray:
    """Same map through the factors: each block as a 4x8 matrix X_m, out = A^T X_m B."""
    X = np.asarray(X, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    a, b = A.shape[0], B.shape[0]
    M, K = X.shape
    Xm = X.reshape(M, K // BLOCK, a, b)
    out = np.einsum("ik,mbij,jl->mbkl", A, Xm, B)
    return out.reshape(M, K)


def rpbh_apply(X, perm, sign) -> np.ndarray:
    """X [M, K] -> X Pi blockdiag(H32/sqrt(32)) D  (permute, block Hadamard, sign)."""
    X = np.asarray(X, dtype=np.float64)
    M, K = X.shape
    perm = np.asarray(perm, dtype=np.int64)
    Xp = X[:, perm]                                              # (x Pi)[j] = x[perm[j]]
    H = sylvester_hadamard(BLOCK) / np.sqrt(BLOCK)
    Xh = (Xp.reshape(M, K // BLOCK, BLOCK) @ H).reshape(M, K)
    return Xh * np.asarray(sign, dtype=np.float64)[None, :]


def fwht(v) -> np.ndarray:
    """Fast Walsh-Hadamard transform along the last axis (unnormalised, Sylvester order).
    Used only as an independent cross-check of ``sylvester_hadamard``."""
    v = np.array(v, dtype=np.float64, copy=True)
    n = v.shape[-1]
    h = 1
    while h < n:
        v = v.reshape(v.shape[:-1] + (n // (2 * h), 2, h))
        a = v[..., 0, :].copy()
        b = v[..., 1, :].copy()
        v[..., 0, :] = a + b
        v[..., 1, :] = a - b
        v = v.reshape(v.shape[:-3] + (n,))
        h *= 2
    return v


def apply(X, T: dict) -> np.ndarray:
    """Online transform Xt = X P for a transform description T (see ``synthetic``)."""
    kind = T["kind"]
    if kind == "kron":
        return kron_apply_explicit(X, T["A"], T["B"])
    if kind == "rpbh":
        return rpbh_apply(X, T["perm"], T["sign"])
    if kind == "none":
        return np.asarray(X, dtype=np.float64).copy()
    raise ValueError(kind)


def inverse_fold(W, T: dict) -> np.ndarray:
    """W' = P^{-1} W for W [K, N] (the offline fold of KroQuant section 01,
    Y = (X P)(P^{-1} W), and of OrbitQuant section 03, W' = R^{-1} W).

    Kron: P^{-1} = blockdiag(A^{-1} (x) B^{-1}) applied to each 32-row block of W.
    RPBH: P is orthogonal, so P^{-1} = P^T = D H^T Pi^T, i.e.
    W' = diag(sign) blockdiag(H/sqrt(32)) W[perm, :].
    """
    W = np.asarray(W, dtype=np.float64)
    K, N = W.shape
    kind = T["kind"]
    if kind == "kron":
        Pinv = np.kron(np.linalg.inv(np.asarray(T["A"], dtype=np.float64)),
                       np.linalg.inv(np.asarray(T["B"], dtype=np.float64)))
        return np.einsum("ij,bjn->bin", Pinv, W.reshape(K // BLOCK, BLOCK, N)).reshape(K, N)
    if kind == "rpbh":
        perm = np.asarray(T["perm"], dtype=np.int64)
        H = sylvester_hadamard(BLOCK) / np.sqrt(BLOCK)
        Wp = W[perm, :].reshape(K // BLOCK, BLOCK, N)
        Wh = np.einsum("ij,bjn->bin", H.T, Wp).reshape(K, N)
        return Wh * np.asarray(T["sign"], dtype=np.float64)[:, None]
    if kind == "none":
        return W.copy()
    raise ValueError(kind)


def forward_fold(L, T: dict) -> np.ndarray:
    """P L for L [K, r]: the map that turns U = Xt L into U = X_c (P L)."""
    L = np.asarray(L, dtype=np.float64)
    K, r = L.shape
    kind = T["kind"]
    if kind == "kron":
        P = kron_block(T["A"], T["B"])
        return np.einsum("ij,bjr->bir", P, L.reshape(K // BLOCK, BLOCK, r)).reshape(K, r)
    if kind == "rpbh":
        # P = Pi H D: (P L)[i] = sum_j Pi[i, j] (H D L)[j];  Pi[i, j] = 1 iff i = perm[j]
        H = sylvester_hadamard(BLOCK) / np.sqrt(BLOCK)
        DL = L * np.asarray(T["sign"], dtype=np.float64)[:, None]
        HDL = np.einsum("ij,bjr->bir", H, DL.reshape(K // BLOCK, BLOCK, r)).reshape(K, r)
        out = np.empty_like(HDL)
        out[np.asarray(T["perm"], dtype=np.int64), :] = HDL
        return out
    if kind == "none":
        return L.copy()
    raise ValueError(kind)


def dense_matrix(T: dict, K: int) -> np.ndarray:
    """The full K x K matrix P (small K only; used by pins)."""
    return apply(np.eye(K), T)
