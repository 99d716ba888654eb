"""The bench's roofline `traffic` comes from the committed ncu record of the
attention kernel: it is the per-head DRAM bytes of the capture scaled to the
workload's heads, and it is withheld (null) once the kernel source differs
from the one that was captured or the workload is another."""

import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _record(path):
    rec = {}
    with open(path) as f:
        for line in f:
            key, sep, val = line.partition(":")
            if sep and not line.startswith("#"):
                rec[key.strip()] = val.strip()
    return rec


def test_committed_record_matches_the_attention_source_and_scales_by_heads():
    b = _bench()
    rec = _record(b.TRAFFIC_FILE)
    assert int(rec["dram_bytes_read"]) + int(rec["dram_bytes_write"]) == int(rec["dram_bytes_per_launch"])
    # the record describes the kernel as committed
    assert rec["source_sha256_16"] == b.source_hash()
    per_head = int(rec["dram_bytes_per_launch"]) / int(rec["heads"])
    assert b.recorded_traffic(rec["workload"], 40) == per_head * 40
    assert b.recorded_traffic(rec["workload"], int(rec["heads"])) == int(rec["dram_bytes_per_launch"])


def test_record_is_withheld_for_another_workload_or_source(tmp_path, monkeypatch):
    b = _bench()
    rec = _record(b.TRAFFIC_FILE)
    assert b.recorded_traffic("10s", 40) is None  # captured on another workload
    # a changed kernel source (another hash): the record no longer describes it
    monkeypatch.setattr(b, "source_hash", lambda path=None: "0" * 16)
    assert b.recorded_traffic(rec["workload"], 40) is None
    # and a missing file gives no figure at all
    monkeypatch.setattr(b, "TRAFFIC_FILE", str(tmp_path / "absent.txt"))
    assert b.recorded_traffic(rec["workload"], 40) is None
