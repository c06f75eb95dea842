"""GPU: kq_linear_noalloc (the layer on the library's built-in workspace) gives the
output of kq_linear with a caller-owned workspace, on consecutive calls that reuse the
built-in workspace with different inputs and sizes, matches the oracle's layer on its
own (fp32 output, 1e-3 relative Frobenius), and refuses a token count whose workspace
would not fit. Named to be collected last, so that it also runs after every other GPU
test has used the library in the same process."""
import numpy as np
import pytest

from oracle import layer as olayer
from tests.kqtest import cached, make_layer, pack_oracle_weights, rel_fro

pytestmark = pytest.mark.gpu


def _linear(kq, L, wbuf, X, out_dtype, noalloc):
    import torch
    M = X.shape[0]
    Y = torch.full((M, L.N), float("nan"), dtype=torch.bfloat16 if out_dtype == kq.OUT_BF16
                   else torch.float32, device="cuda")
    if noalloc:
        kq.linear_noalloc(L, wbuf, X, Y, out_dtype)
    else:
        act = torch.empty(kq.act_bytes(L, M), dtype=torch.uint8, device="cuda")
        kq.linear(L, wbuf, X, Y, act, out_dtype)
        torch.cuda.synchronize()
        assert kq.last_device_error(L, act, M) == 0
    torch.cuda.synchronize()
    return Y.float().cpu().double().numpy()


@pytest.mark.parametrize("index,kw", [(3, dict(M=300, N=768)), (2, dict(M=515, N=1024))],
                         ids=["kron-centre", "rpbh"])
def test_noalloc_matches_linear_on_consecutive_calls(cuda_device, index, kw):
    import torch
    import w4a4_post_quantization_token_b200 as kq
    w, inp, prep = cached(index, **kw)
    L = make_layer(w, inp["T"])
    wbuf = pack_oracle_weights(L, prep)
    X = inp["X"].cuda()
    # a second input of another size and values: the built-in workspace then holds the
    # first call's larger contents when the second call runs
    g = torch.Generator().manual_seed(11)
    X2 = (inp["X"][: w.M // 2].float() * (1 + torch.rand(w.M // 2, 1, generator=g))).to(
        torch.bfloat16).cuda()
    for out in (kq.OUT_F32, kq.OUT_BF16):
        tol = 1e-3 if out == kq.OUT_F32 else 4e-3
        for Xi in (X, X2, X):
            ref = _linear(kq, L, wbuf, Xi, out, noalloc=False)
            got = _linear(kq, L, wbuf, Xi, out, noalloc=True)
            assert np.all(np.isfinite(got))
            assert rel_fro(got, ref) <= tol
            if out == kq.OUT_F32:
                # and on its own against the oracle's fp64 layer
                Yo = olayer.linear(Xi.cpu(), inp["T"], w.center, prep)
                assert rel_fro(got, Yo) <= 1e-3


def test_noalloc_rejects_too_large_M(cuda_device):
    import torch
    import w4a4_post_quantization_token_b200 as kq
    w, inp, prep = cached(3, M=300, N=768)
    L = make_layer(w, inp["T"])
    M = 1
    while kq.act_bytes(L, M) <= kq.NOALLOC_WORKSPACE_BYTES:
        M *= 2
    assert kq.lib.kq_linear_noalloc(L.desc, 256, 256, M, 256, kq.OUT_F32, None) == 5
    # the largest M that fits is accepted
    lo, hi = M // 2, M
    while hi - lo > 1:
        mid = (lo + hi) // 2
        lo, hi = (mid, hi) if kq.act_bytes(L, mid) <= kq.NOALLOC_WORKSPACE_BYTES else (lo, mid)
    wbuf = pack_oracle_weights(L, prep)
    X = torch.zeros((lo, L.K), dtype=torch.bfloat16, device="cuda")
    Y = torch.empty((lo, L.N), dtype=torch.float32, device="cuda")
    kq.linear_noalloc(L, wbuf, X, Y)
    torch.cuda.synchronize()
    assert torch.count_nonzero(Y).item() == 0
