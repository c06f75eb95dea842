"""Host logic of bench.py (CPU): the DRAM-traffic lookup that fills `roofline.traffic`.

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
