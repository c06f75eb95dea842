"""GPU: the block-scaled FP4 GEMM (kq_gemm) on inputs whose MXFP4 encoding is exact.

Activation and weight blocks hold E2M1 grid values times one power of two per block,
so the fp64 product of the decoded operands is exact and the kernel may differ only by
fp32 accumulation rounding. This pins the operand layouts (nibble order, K-major
tiles, the 128x4 scale-factor layout and its TMEM mapping, scale byte ids) and the
fused low-rank (U L2) and rank-1 (mu s) terms."""
import numpy as np
import pytest

from oracle import mxfp4
from synthetic import exact_grid_inputs
from tests.kqtest import pack_nibbles

pytestmark = pytest.mark.gpu


def _run(M, K, N, rank=0, center=False, out_bf16=False, seed=0):
    import torch
    import w4a4_post_quantization_token_b200 as kq
    Xq, Wq = exact_grid_inputs(M, K, N, seed)
    Xq, Wq = Xq.astype(np.float64), Wq.astype(np.float64)
    xc, xs = mxfp4.encode(Xq)
    wc, wsc = mxfp4.encode(Wq)
    np.testing.assert_array_equal(mxfp4.decode(xc, xs), Xq)     # exact by construction
    rng = np.random.default_rng(seed + 1)
    L = kq.Layer(K, N, rank, center, {"kind": "none"})
    s = rng.standard_normal(N).astype(np.float32)
    mu = rng.standard_normal(M).astype(np.float32) * 3 if center else None
    if rank:
        U = torch.randn(M, rank, dtype=torch.float32).to(torch.float16)
        L2 = torch.randn(rank, N, dtype=torch.float32).to(torch.bfloat16)
        L1p = torch.zeros(K, rank, dtype=torch.float32)
    else:
        U = L2 = L1p = None
    wbuf = torch.empty(kq.weights_bytes(L), dtype=torch.uint8, device="cuda")
    kq.weights_pack(L, torch.from_numpy(pack_nibbles(wc)).cuda(), torch.from_numpy(wsc).cuda(),
                    L1p.cuda() if rank else None, L2.cuda() if rank else None,
                    torch.from_numpy(s).cuda(), wbuf)
    act = torch.empty(kq.act_bytes(L, M), dtype=torch.uint8, device="cuda")
    kq.act_pack(L, torch.from_numpy(pack_nibbles(xc)).cuda(), torch.from_numpy(xs).cuda(),
                torch.from_numpy(mu).cuda() if center else None, U.cuda() if rank else None, M, act)
    Y = torch.empty((M, N), dtype=torch.bfloat16 if out_bf16 else torch.float32, device="cuda")
    kq.gemm(L, wbuf, act, M, Y, kq.OUT_BF16 if out_bf16 else kq.OUT_F32)
    torch.cuda.synchronize()
    assert kq.last_device_error(L, act, M) == 0
    ref = Xq @ Wq.T
    absref = np.abs(Xq) @ np.abs(Wq).T
    if rank:
        Ud, L2d = U.double().numpy(), L2.double().numpy()
        ref = ref + Ud @ L2d
        absref = absref + np.abs(Ud) @ np.abs(L2d)
    if center:
        ref = ref + np.outer(mu.astype(np.float64), s.astype(np.float64))
        absref = absref + np.abs(np.outer(mu, s))
    return Y.float().cpu().double().numpy(), ref, absref


@pytest.mark.parametrize("M,K,N", [(128, 256, 256), (200, 1152, 384), (300, 1152, 512),
                                   (1, 32, 16), (129, 96, 48), (256, 3072, 256), (64, 12288, 256)])
def test_exact_grid_product(cuda_device, M, K, N):
    Y, ref, absref = _run(M, K, N)
    assert np.all(np.abs(Y - ref) <= 1e-5 * absref + 1e-30)


@pytest.mark.parametrize("rank", [1, 17, 32, 64])
def test_lowrank_branch_fused(cuda_device, rank):
    Y, ref, absref = _run(160, 640, 512, rank=rank)
    assert np.all(np.abs(Y - ref) <= 1e-5 * absref + 1e-30)


def test_rank1_mean_restore_fused(cuda_device):
    Y, ref, absref = _run(257, 512, 768, rank=16, center=True)
    assert np.all(np.abs(Y - ref) <= 1e-5 * absref + 1e-30)


def test_bf16_output(cuda_device):
    Y, ref, absref = _run(130, 512, 256, rank=8, center=True, out_bf16=True)
    assert np.all(np.abs(Y - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5 * absref + 1e-30)


def test_per_block_scale_perturbation(cuda_device):
    """Changing one activation block's scale by 2^k changes only that block's contribution:
    checks that each scale byte reaches exactly its own 32 elements."""
    import torch
    import w4a4_post_quantization_token_b200 as kq
    M, K, N = 256, 512, 256
    Xq, Wq = exact_grid_inputs(M, K, N, 5)
    xc, xs = mxfp4.encode(Xq.astype(np.float64))
    wc, wsc = mxfp4.encode(Wq.astype(np.float64))
    rng = np.random.default_rng(9)
    xs2 = xs.copy()
    rows = rng.integers(0, M, 40)
    blks = rng.integers(0, K // 32, 40)
    xs2[rows, blks] = np.clip(xs2[rows, blks].astype(int) + rng.integers(-3, 4, 40), 1, 250)
    L = kq.Layer(K, N, 0, False, {"kind": "none"})
    wbuf = torch.empty(kq.weights_bytes(L), dtype=torch.uint8, device="cuda")
    kq.weights_pack(L, torch.from_numpy(pack_nibbles(wc)).cuda(), torch.from_numpy(wsc).cuda(),
                    None, None, torch.zeros(N).cuda(), wbuf)
    act = torch.empty(kq.act_bytes(L, M), dtype=torch.uint8, device="cuda")
    kq.act_pack(L, torch.from_numpy(pack_nibbles(xc)).cuda(), torch.from_numpy(xs2).cuda(), None,
                None, M, act)
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    kq.gemm(L, wbuf, act, M, Y)
    torch.cuda.synchronize()
    Xd = mxfp4.decode(xc, xs2)
    Wd = mxfp4.decode(wc, wsc)
    ref = Xd @ Wd.T
    absref = np.abs(Xd) @ np.abs(Wd).T
    assert np.all(np.abs(Y.cpu().double().numpy() - ref) <= 1e-5 * absref + 1e-30)
