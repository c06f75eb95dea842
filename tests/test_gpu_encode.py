"""GPU: the MXFP4 encoder alone (kq_debug_encode_f32) is bit-exact against the oracle
encoder when both are fed the same float32 values (OCP MX v1.0 rule; KroQuant
commentary section 03 names MXFP4)."""
import numpy as np
import pytest

from oracle import mxfp4
from tests.kqtest import pack_nibbles
from tests.test_oracle_mxfp4 import load_golden

pytestmark = pytest.mark.gpu


def gpu_encode(V: np.ndarray):
    import torch
    import w4a4_post_quantization_token_b200 as kq
    M, K = V.shape
    Vt = torch.from_numpy(np.ascontiguousarray(V, dtype=np.float32)).cuda()
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((M, K // 32), dtype=torch.uint8, device="cuda")
    kq.debug_encode_f32(Vt, codes, scales)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


def check_exact(V):
    V = np.asarray(V, dtype=np.float32).astype(np.float64)
    oc, os_ = mxfp4.encode(V)
    gc, gs = gpu_encode(V)
    np.testing.assert_array_equal(gs, os_)
    np.testing.assert_array_equal(gc, pack_nibbles(oc))


def test_golden_blocks(cuda_device):
    cases = load_golden()
    V = np.stack([c["values"] for c in cases])
    gc, gs = gpu_encode(V)
    for i, c in enumerate(cases):
        assert int(gs[i, 0]) == c["scale"], c["name"]
        np.testing.assert_array_equal(gc[i], pack_nibbles(c["codes"][None, :])[0], err_msg=c["name"])


def test_random_and_heavy_tailed(cuda_device):
    rng = np.random.default_rng(11)
    V = rng.standard_normal((512, 1024)) * np.exp2(rng.integers(-30, 30, size=(512, 1)))
    V = np.where(rng.random(V.shape) < 0.05, rng.standard_t(2, V.shape) * 40, V)
    check_exact(V)


def test_adversarial_ties_and_subnormals(cuda_device):
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    mids = (grid[1:] + grid[:-1]) / 2
    rows = []
    for e in (-127, -126, -100, -3, 0, 7, 60, 124):
        base = np.concatenate([[6.0], mids, -mids, grid[1:], [7.99, -6.5, 5.0000001, 0.0, -0.0]])
        rows.append(np.pad(base, (0, 64 - len(base))) * 2.0 ** e)
    for k in range(-149, 127, 3):
        p = 2.0 ** k
        rows.append(np.array([p, p / 2, p * 0.75, p * 0.375, -p * 0.1875, p * (1 - 2 ** -23)] +
                             [0.0] * 58))
    V = np.array(rows, dtype=np.float64).astype(np.float32).astype(np.float64)
    check_exact(V)


def test_negative_zero_and_all_zero_blocks(cuda_device):
    V = np.zeros((4, 64))
    V[1, :] = -0.0
    V[2, 3] = -1e-30
    V[2, 0] = 1.0
    V[3, :32] = -0.0
    V[3, 40] = -3.0
    check_exact(V)


def test_exhaustive_bf16_patterns(cuda_device):
    bits = np.arange(65536, dtype=np.uint32)
    vals = (bits << 16).view(np.float32).astype(np.float64)
    vals = vals[np.isfinite(vals)]
    vals = np.concatenate([vals, np.zeros((-len(vals)) % 8)])
    blocks = np.zeros((len(vals), 32))
    blocks[:, 0] = vals
    blocks[:, 1] = 1.0
    check_exact(blocks.reshape(-1, 256))
    alone = np.zeros((len(vals), 32))
    alone[:, 5] = vals
    check_exact(alone.reshape(-1, 128))
