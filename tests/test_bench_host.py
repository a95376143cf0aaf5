"""Host logic of bench.py that needs no GPU: the DRAM-traffic lookup is keyed
to the kernel sources, so a capture never outlives the code it measured."""
import json
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402


def test_traffic_entry_follows_the_kernel_sources(tmp_path, monkeypatch):
    f = tmp_path / "traffic.json"
    f.write_text(json.dumps({
        "w": {"kernel_source_sha": bench.kernel_source_sha(), "dram_bytes_per_launch": 123},
        "stale": {"kernel_source_sha": "0" * 16, "dram_bytes_per_launch": 456},
        "prologue:w": {"kernel_source_sha": bench.kernel_source_sha(bench.PROLOGUE_SOURCES),
                       "dram_bytes_per_launch": 789},
    }))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.traffic_per_launch("w") == 123
    assert bench.traffic_per_launch("stale") is None
    assert bench.traffic_per_launch("missing") is None
    assert bench.captured_traffic("prologue:w", bench.PROLOGUE_SOURCES) == 789
    # the prologue's entry is keyed to its own source, not the attention kernel's
    assert bench.captured_traffic("prologue:w") is None


def test_source_hash_changes_with_the_source(tmp_path, monkeypatch):
    a = tmp_path / "k.cuh"
    a.write_text("x")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h1 = bench.kernel_source_sha(["k.cuh"])
    a.write_text("y")
    assert bench.kernel_source_sha(["k.cuh"]) != h1
