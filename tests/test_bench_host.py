"""Host logic of bench.py (no GPU): the workload registry and the gate that reports DRAM traffic from
a committed ncu capture only while the kernel source is the one the counters were taken on."""
import hashlib
import json
import os

import bench


def test_registry_is_consistent():
    assert bench.DEFAULT_WORKLOAD in bench.WORKLOADS
    for name, spec in bench.WORKLOADS.items():
        assert spec["kind"] in bench.METRICS, name
        assert spec["d"] in (64, 128), name
    # the headline runs the forward at the full length
    assert bench.WORKLOADS[bench.DEFAULT_WORKLOAD]["kind"] == "sa_fwd"


def test_committed_traffic_entries_name_real_workloads_and_sources():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        tr = json.load(f)
    for workload, per_norm in tr.items():
        if workload == "note":
            continue
        assert workload in bench.WORKLOADS, workload
        for norm, entry in per_norm.items():
            assert norm in ("proto", "token", "stca"), (workload, norm)
            assert os.path.exists(os.path.join(bench.ROOT, entry["source"])), entry["source"]
            assert entry["bytes"] > 0 and len(entry["source_sha256"]) == 16


def test_traffic_gate_follows_the_source_hash(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("// kernel v1\n")
    digest = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"w": {"proto": {"bytes": 1234, "kernel": "k", "source": "kernel.cu", "source_sha256": digest}}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_for("w", "proto") == 1234
    assert bench.traffic_for("w", "token") is None      # no capture for this normalisation
    assert bench.traffic_for("other", "proto") is None  # no capture for this workload
    src.write_text("// kernel v2\n")                     # the kernel changed since the capture
    assert bench.traffic_for("w", "proto") is None


def test_traffic_gate_without_captures(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_for(bench.DEFAULT_WORKLOAD, "proto") is None
