"""GPU: behaviour at the C-ABI boundary (include/kq.h conventions).

* Device pointers need only a 16-byte boundary (what a TMA global address needs): the
  whole layer runs on X, Y, workspace and weights that sit 16 bytes past a 256-byte
  boundary and matches the oracle at the layer tolerance (1e-3 relative Frobenius, fp32
  output).
* Bounded device waits: a wait that nothing completes runs out after its limit, the
  error word reports KQ_ERR_DEVICE_TIMEOUT, and the context stays usable (an ordinary
  layer call afterwards matches the oracle). The failure is made on purpose with a
  barrier nobody arrives on: no fault, no trap, no unbounded wait.
* The 16-bit low-rank branch (SVDQuant explainer, section 3) holds U as fp16: a token
  whose U leaves the fp16 range is saturated and reported as KQ_ERR_LOWRANK_RANGE
  instead of returning a wrong output with status OK."""
import numpy as np
import pytest

from oracle import layer as olayer
from tests.kqtest import cached, make_layer, pack_oracle_weights, rel_fro

pytestmark = pytest.mark.gpu


def _at_offset(nbytes: int, offset: int):
    """A uint8 device view of nbytes that starts `offset` bytes past a 256-byte boundary."""
    import torch
    base = torch.empty(nbytes + 512, dtype=torch.uint8, device="cuda")
    skip = (-base.data_ptr()) % 256 + offset
    v = base[skip:skip + nbytes]
    assert v.data_ptr() % 256 == offset
    return v


def test_linear_on_buffers_at_a_16_byte_offset(cuda_device):
    import torch
    import w4a4_post_quantization_token_b200 as kq
    w, inp, prep = cached(3, M=300, N=256)            # Kronecker, centred, rank 32
    L = make_layer(w, inp["T"])
    wb0 = pack_oracle_weights(L, prep)
    wbuf = _at_offset(wb0.numel(), 16)
    wbuf.copy_(wb0)
    X = _at_offset(w.M * w.K * 2, 16).view(torch.bfloat16).view(w.M, w.K)
    X.copy_(inp["X"].cuda())
    Y = _at_offset(w.M * w.N * 4, 16).view(torch.float32).view(w.M, w.N)
    act = _at_offset(kq.act_bytes(L, w.M), 16)
    kq.linear(L, wbuf, X, Y, act, kq.OUT_F32)
    torch.cuda.synchronize()
    assert kq.last_device_error(L, act, w.M) == 0
    Yref = olayer.linear(inp["X"], inp["T"], w.center, prep)
    err = rel_fro(Y.double().cpu().numpy(), Yref)
    assert err <= 1e-3, err
    # an 8-byte offset is refused before anything is launched
    bad = _at_offset(w.M * w.N * 4, 8).view(torch.float32)
    r = kq.lib.kq_linear(L.desc, wbuf.data_ptr(), X.data_ptr(), w.M, bad.data_ptr(), kq.OUT_F32,
                         act.data_ptr(), act.numel(), torch.cuda.current_stream().cuda_stream)
    assert r == 3


def test_bounded_wait_runs_out_and_the_context_stays_usable(cuda_device):
    import time

    import torch
    import w4a4_post_quantization_token_b200 as kq
    w, inp, prep = cached(1, M=160, N=512)
    L = make_layer(w, inp["T"])
    act = torch.empty(kq.act_bytes(L, w.M), dtype=torch.uint8, device="cuda")
    act.zero_()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    kq.debug_wait_timeout(L, act, w.M, 2000)                  # 2 ms limit
    assert kq.last_device_error(L, act, w.M) == kq.ERR_DEVICE_TIMEOUT
    elapsed = time.perf_counter() - t0
    assert 0.002 <= elapsed < 5.0, elapsed
    # the word is cleared by the read
    assert kq.last_device_error(L, act, w.M) == 0
    # and the device still runs the layer correctly
    wbuf = pack_oracle_weights(L, prep)
    Y = torch.empty((w.M, w.N), dtype=torch.float32, device="cuda")
    kq.linear(L, wbuf, inp["X"].cuda(), Y, act, kq.OUT_F32)
    torch.cuda.synchronize()
    assert kq.last_device_error(L, act, w.M) == 0
    Yref = olayer.linear(inp["X"], inp["T"], w.center, prep)
    assert rel_fro(Y.double().cpu().numpy(), Yref) <= 1e-3


def test_lowrank_overflow_is_reported(cuda_device):
    """One token scaled so that its low-rank activation U = Xt L1 leaves the fp16 range:
    the call reports KQ_ERR_LOWRANK_RANGE. The same batch without it reports nothing, and
    its other rows still match the oracle row by row (the saturation touches only the
    offending token's U)."""
    import torch
    import w4a4_post_quantization_token_b200 as kq
    w, inp, prep = cached(3, M=300, N=256)
    L = make_layer(w, inp["T"])
    wbuf = pack_oracle_weights(L, prep)
    Xh = inp["X"].clone()
    big = 7
    # |U| of this row ~ 2e4 * |Xt L1| / |X| for the workload's typical tokens: far past 65504
    Xh[big] = (Xh[big].float() * 2.0e4).to(torch.bfloat16)
    U_big = olayer.quantize_act(Xh[big:big + 1], inp["T"], w.center, prep)["U"]
    assert np.max(np.abs(U_big)) > 65504.0
    act = torch.empty(kq.act_bytes(L, w.M), dtype=torch.uint8, device="cuda")
    Y = torch.empty((w.M, w.N), dtype=torch.float32, device="cuda")
    kq.linear(L, wbuf, Xh.cuda(), Y, act, kq.OUT_F32)
    assert kq.last_device_error(L, act, w.M) == kq.ERR_LOWRANK_RANGE
    Yref = olayer.linear(Xh, inp["T"], w.center, prep)
    Yg = Y.double().cpu().numpy()
    keep = np.arange(w.M) != big
    assert rel_fro(Yg[keep], Yref[keep]) <= 1e-3
    kq.linear(L, wbuf, inp["X"].cuda(), Y, act, kq.OUT_F32)
    assert kq.last_device_error(L, act, w.M) == 0
