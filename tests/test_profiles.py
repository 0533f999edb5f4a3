"""The committed ncu figures the bench reports: each DRAM-traffic entry names its summary and its sources, and the
bench reports it only while those sources are unchanged since the capture."""

import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _entries():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        return json.load(f)


def test_every_traffic_entry_has_its_summary_and_sources():
    for name, e in _entries().items():
        assert os.path.exists(os.path.join(ROOT, e["profile"])), (name, e["profile"])
        for src in e["sources"]:
            assert os.path.exists(os.path.join(ROOT, "sparse_long_context_lightning_b200", "csrc", src)), (name, src)
        assert e["dram_bytes_per_launch"] == e["dram_read"] + e["dram_write"], name
        assert e["dram_bytes_per_launch"] > 0, name


def test_committed_traffic_is_reported_exactly_while_the_sources_match():
    import bench

    for name, e in _entries().items():
        current = bench.kernel_source_hash(e["sources"]) == e["source_hash"]
        assert bench.committed_traffic(name) == (e["dram_bytes_per_launch"] if current else None), name


def test_committed_traffic_is_withheld_when_the_source_changed(monkeypatch):
    import bench

    assert bench.committed_traffic("no_such_kernel") is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda sources: "0000000000000000")
    for name in _entries():
        assert bench.committed_traffic(name) is None
