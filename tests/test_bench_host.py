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


def _traffic_file(bench, tmp_path, workload="varlen64k"):
    t = {"workload": workload}
    for stage, files, b in (("attn_bwd", ["attn_bwd_sm100.cu", "common.cuh"], 123),
                            ("attn_fwd", ["attn_fwd_sm100.cu", "sm100.cuh"], 456)):
        t[stage] = {"bytes": b, "sources": files, "source_sha256": bench.kernel_source_hash(files)}
    p = tmp_path / "traffic.json"
    p.write_text(json.dumps(t))
    return str(p)


def test_stored_traffic_matches_current_sources(tmp_path):
    bench = _bench()
    p = _traffic_file(bench, tmp_path)
    assert bench.stored_traffic("varlen64k", "attn_bwd", p) == 123
    assert bench.stored_traffic("varlen64k", "attn_fwd", p) == 456
    assert bench.stored_traffic("single64k", "attn_fwd", p) is None          # other workload
    assert bench.stored_traffic("varlen64k", "no_such_stage", p) is None


def test_stored_traffic_goes_null_when_a_source_changes(tmp_path, monkeypatch):
    bench = _bench()
    p = _traffic_file(bench, tmp_path)
    monkeypatch.setattr(bench, "kernel_source_hash", lambda files: "0" * 64)
    assert bench.stored_traffic("varlen64k", "attn_bwd", p) is None


def test_committed_traffic_file_is_well_formed():
    bench = _bench()
    with open(bench.TRAFFIC_FILE) as f:
        t = json.load(f)
    for stage in ("attn_bwd", "attn_fwd"):
        assert t[stage]["bytes"] > 0 and t[stage]["sources"] and len(t[stage]["source_sha256"]) == 64
