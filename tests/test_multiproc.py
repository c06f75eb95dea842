"""Multi-process host logic on CPU (gloo, world size 2): the max-over-ranks timing that
bench.py reports for N GPUs, the row split of a global batch, and the property that makes
the path shard without a collective: token rows are independent, so each rank's rows
through the layer, gathered, equal the whole batch through it (oracle, float64)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, fn, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        q.put((rank, fn(rank, world)))
    finally:
        dist.destroy_process_group()


def _run(fn, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, fn, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return out


def _timing(rank, world):
    import bench
    return bench.max_over_ranks(10.0 + 7.5 * rank, dist, "cpu")


def test_max_over_ranks():
    out = _run(_timing)
    assert out == {0: 17.5, 1: 17.5}


def test_shard_rows_cover_the_batch():
    import bench
    for M in (1, 7, 4096, 35100):
        for world in (1, 2, 3, 8):
            spans = [bench.shard_rows(M, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == M
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [e - b for b, e in spans]
            assert max(sizes) - min(sizes) <= 1


def _sharded_layer(rank, world):
    import bench
    from oracle import layer as olayer
    from synthetic import make_inputs, workload
    w = workload(1, M=70, N=96)
    inp = make_inputs(w)
    prep = olayer.prepare(inp["W"], inp["T"], w.rank)
    b, e = bench.shard_rows(w.M, rank, world)
    Y = torch.from_numpy(olayer.linear(inp["X"][b:e], inp["T"], w.center, prep))
    sizes = [bench.shard_rows(w.M, r, world) for r in range(world)]
    parts = [torch.zeros((s[1] - s[0], w.N), dtype=torch.float64) for s in sizes]
    dist.all_gather(parts, Y)
    gathered = torch.cat(parts).numpy()
    full = olayer.linear(inp["X"], inp["T"], w.center, prep)
    return float(np.max(np.abs(gathered - full)) / np.max(np.abs(full)))


def test_token_sharding_needs_no_exchange():
    out = _run(_sharded_layer)
    assert all(v <= 1e-12 for v in out.values()), out
