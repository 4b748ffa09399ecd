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
            assert norm in ("proto", "token", "stca", "refine", "stca_bwd"), (workload, norm)
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


def test_launcher_command_starts_one_process_per_gpu():
    cmd = bench.launcher_command(4, ["--gpus", "4", "--steps", "3"])
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--master-addr=127.0.0.1" in cmd
    assert cmd[-5:] == [os.path.join(bench.ROOT, "bench.py"), "--gpus", "4", "--steps", "3"]


def test_rank_users_partition_the_global_batch():
    """Weak scaling: N ranks split N copies of the workload's users, balanced by valid length, and
    one rank alone gets exactly the workload."""
    for name in ("sa_fwd_b64_ragged_h4_d64_k256", "sa_fwd_b8_l100k_h8_d128_k512_masked", "sa_fwd_paper_h1_d128_k1024"):
        spec = bench.WORKLOADS[name]
        one, su1 = bench.rank_users(spec, 0, 1)
        assert one == bench.lengths_for(spec["lens"]) and su1 == spec["seqused"]
        for world in (2, 4, 8):
            parts = [bench.rank_users(spec, r, world) for r in range(world)]
            lens = [x for p, _ in parts for x in p]
            assert sorted(lens) == sorted(bench.lengths_for(spec["lens"], world))
            valid = [sum(min(a, b) for a, b in zip(p, su)) if su else sum(p) for p, su in parts]
            assert max(valid) - min(valid) <= max(bench.lengths_for(spec["lens"], world)), (name, world, valid)
            per_rank = sum(valid) / world
            assert max(valid) <= 1.15 * per_rank, (name, world, valid)


def test_gpus_flag_launches_ranks_on_the_cpu():
    """`bench.py --gpus 2` outside a launcher re-executes itself under torch.distributed.run; the
    reference arm (the oracle, no GPU) then prints one line from rank 0 with n_gpus 2."""
    import subprocess
    import sys
    out = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--gpus", "2", "--impl", "reference",
                          "--steps", "1", "--warmup", "3", "--ref-seconds", "0.2",
                          "--workload", "stca_b16_t512_h4_d64_l10k_s256"],
                         capture_output=True, text=True, timeout=600, cwd=bench.ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(x) for x in out.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1 and lines[0]["n_gpus"] == 2 and lines[0]["impl"] == "reference"
