"""Host-side logic of bench.py (no GPU): the stored ncu traffic is reported
only for the workload it was measured on and only while the kernel sources it
describes are unchanged."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    sys.path.insert(0, ROOT)
    argv, sys.argv = sys.argv, ["bench.py"]
    try:
        import bench
    finally:
        sys.argv = argv
    return bench


def test_stored_traffic_matches_current_sources():
    bench = _bench()
    with open(os.path.join(ROOT, "profiles", "roofline_traffic.json")) as f:
        t = json.load(f)
    for stage in ("attn_bwd", "attn_fwd"):
        assert bench.stored_traffic("varlen64k", stage) == t[stage]["bytes"]
        assert bench.stored_traffic("single64k", stage) is None          # other workload
    assert bench.stored_traffic("varlen64k", "no_such_stage") is None


def test_stored_traffic_goes_null_when_a_source_changes(tmp_path, monkeypatch):
    bench = _bench()
    real = bench.kernel_source_hash
    monkeypatch.setattr(bench, "kernel_source_hash", lambda files: "0" * 64 if files else real(files))
    assert bench.stored_traffic("varlen64k", "attn_bwd") is None
