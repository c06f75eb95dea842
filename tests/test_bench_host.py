"""Host logic of bench.py (CPU): the DRAM-traffic lookup that fills `roofline.traffic`, and
the algorithmic work per step that the roofline fractions divide by.

A record applies only to its own (kernel, workload) pair and only while the kernel's
sources hash to the recorded digest; otherwise the bench reports null rather than a figure
taken on other code. Also checks that every committed record still matches the sources in
the tree (a record left stale by a kernel change would silently drop out of the bench)."""
import hashlib
import json
import os

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _digest(root, srcs):
    h = hashlib.sha256()
    for s in srcs:
        with open(os.path.join(root, s), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


@pytest.fixture
def fake_root(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "src").mkdir()
    (tmp_path / "src" / "k.cu").write_text("kernel v1\n")
    rec = {"kernel": "k_x", "workload": "w M=1", "sources": ["src/k.cu"],
           "source_sha256_16": _digest(tmp_path, ["src/k.cu"]),
           "dram_read_bytes": 1000, "dram_write_bytes": 24, "note": "n", "profile": "p.md"}
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps({"records": [rec]}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return tmp_path


def test_traffic_matches_kernel_and_workload(fake_root):
    got = bench.measured_traffic("k_x", "w M=1")
    assert got is not None and got["bytes"] == 1024
    assert bench.measured_traffic("k_x", "w M=2") is None
    assert bench.measured_traffic("k_y", "w M=1") is None


def test_traffic_dropped_when_source_changes(fake_root):
    (fake_root / "src" / "k.cu").write_text("kernel v2\n")
    assert bench.measured_traffic("k_x", "w M=1") is None


def test_traffic_missing_file(fake_root):
    os.remove(fake_root / "profiles" / "dram_traffic.json")
    assert bench.measured_traffic("k_x", "w M=1") is None


def test_committed_records_match_tree():
    with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
        recs = json.load(f)["records"]
    assert recs
    for r in recs:
        assert _digest(ROOT, r["sources"]) == r["source_sha256_16"], r["kernel"]
        assert r["dram_read_bytes"] > 0 and os.path.exists(os.path.join(ROOT, r["profile"]))


def test_algorithmic_work_video_dit():
    """The roofline numerators of the video-DiT layer (35100 x 3072 -> 3072, centred, r = 64),
    as the bench lines report them (`algorithmic_per_launch`)."""
    flops, gbytes, qbytes = bench.algorithmic_work(35100, 3072, 3072, 64, True)
    assert flops == 676_400_025_600          # 2MNK + 2MNr + MN
    assert qbytes == 277_570_800             # X + codes + scales + means + U
    # codes 53.9 MB + residual 4.7 MB + scales 3.7 MB + U 4.5 MB + L2 0.4 MB + s, mu + Y 215.7 MB
    assert gbytes == 282_989_808


def test_algorithmic_work_terms():
    M, K, N = 256, 1024, 512
    f0, g0, q0 = bench.algorithmic_work(M, K, N, 0, False)
    assert f0 == 2 * M * N * K
    assert q0 == M * K * 2 + M * K / 2 + M * K / 32 + M * 4          # no U without a low-rank branch
    f1, g1, q1 = bench.algorithmic_work(M, K, N, 5, True)
    assert f1 - f0 == 2 * M * N * 5 + M * N                          # rank-5 branch + rank-1 restore
    assert q1 - q0 == M * 64 * 2                                     # U stored 64 wide
    assert g1 - g0 == (M + N) * 64 * 2 + M * 4                       # U, L2 and the means
    _, g32, _ = bench.algorithmic_work(M, K, N, 0, False, out_bf16=False)
    assert g32 - g0 == M * N * 2                                     # fp32 Y instead of bf16
    _, glut, qlut = bench.algorithmic_work(M, K, N, 0, False, lut=True)
    assert glut - g0 == (M + N) * K * 2 - (M + N) * K / 2 - (M + N) * K / 32   # fp16 operands, no scales
    assert qlut == M * K * 2 + M * K * 2 + M * 8                     # fp16 operand out, mean and sigma
