#!/usr/bin/env python
"""Benchmark of the FlashSA forward (Sketch Attention, SequenceO1 §3.1 / §4.4) on B200.

Default workload: 8 users x 100,000 history tokens, H=8 heads, d=128, k=512 prototypes,
prototype-wise normalisation (the paper's Eq. (8)), bf16 inputs, fp32 sketch and per-token lse.
One step = one sa_forward call (schedule, fused kernel, partial combine, lse padding fill).

  python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--norm proto|token]
  python bench.py --impl reference ...   # the fp64 CPU oracle on a bounded sample

Multi-GPU (torchrun, one process per GPU): every rank runs its own batch of the workload
(independent users, no collective on the data path) -> weak scaling; the reported time is the
max over ranks of the device-timed region.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SA fwd history-tokens/s and TFLOP/s (fraction of B200 bf16 peak) at L=100K"
UNIT = "history-tokens/s"

# name -> (lengths or "ragged64", H, d, k, seqused, q_sigma_is_inv_sqrt_d)
WORKLOADS = {
    "sa_fwd_b8_l100k_h8_d128_k512": ([100_000] * 8, 8, 128, 512, None),
    "sa_fwd_b8_l100k_h8_d128_k512_masked": ([100_000] * 8, 8, 128, 512, [70_000] + [100_000] * 7),
    "sa_fwd_b64_ragged_h4_d64_k256": ("ragged64", 4, 64, 256, None),
    "sa_fwd_paper_h1_d128_k1024": ("paper", 1, 128, 1024, None),
    # profiling size: same per-tile work as the headline, 205 MB of K+V (> L2), ~0.25 ms
    "sa_fwd_b2_l100k_h2_d128_k512": ([100_000] * 2, 2, 128, 512, None),
}
DEFAULT_WORKLOAD = "sa_fwd_b8_l100k_h8_d128_k512"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": pk["hbm_gbs"], "bf16_tflops": pk["bf16_tflops"],
                "bf16_tflops_sustained": pk.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def lengths_for(spec, rank):
    if isinstance(spec, list):
        return spec
    rng = np.random.default_rng(1 if spec == "ragged64" else 5)
    if spec == "ragged64":
        x = np.exp(rng.uniform(math.log(1000), math.log(100_000), 64))
        return [int(v) for v in np.clip(np.round(x), 1000, 100_000)]
    return [int(v) for v in np.clip(np.round(rng.normal(85_000, 10_000, 8)), 1000, 100_000)]


def make_device_inputs(name, rank, device):
    """Seeded synthetic inputs drawn on the device: K, V ~ N(0,1), Q ~ N(0,1)/sqrt(d), bf16."""
    import torch
    spec, H, d, kp, su = WORKLOADS[name]
    lens = lengths_for(spec, rank)
    T = sum(lens)
    gen = torch.Generator(device=device)
    gen.manual_seed(1000 + rank)
    q = (torch.randn((H, kp, d), generator=gen, device=device) / math.sqrt(d)).bfloat16()
    k = torch.randn((T, H, d), generator=gen, device=device, dtype=torch.bfloat16)
    v = torch.randn((T, H, d), generator=gen, device=device, dtype=torch.bfloat16)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32), device=device)
    seqused = torch.tensor(np.array(su, dtype=np.int32), device=device) if su else None
    valid = sum(min(a, b) for a, b in zip(lens, su)) if su else T
    return dict(q=q, k=k, v=v, cu=cu, seqused=seqused, lens=lens, H=H, d=d, k_protos=kp, valid=valid,
                users=len(lens), scale=1.0)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during the timed region."""
    Q = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(", ") for r in out.strip().splitlines() if r.strip()]
        mine = [r for r in rows if len(r) >= 10 and (self.uuid is None or self.uuid in r[1])]
        if not mine:
            mine = [r for r in rows if len(r) >= 10]
        if not mine:
            return None
        sm = [float(r[2]) for r in mine if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in mine if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in mine for i in range(4) if r[6 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(mine)}


def cpu_baseline(inp, budget_s=12.0):
    """The fp64 oracle (oracle/sa.py, as it stands) on whole (user, head) problems of the same
    workload until about budget_s seconds of CPU work; returns history-tokens/s equivalents."""
    import torch
    import oracle
    from threadpoolctl import threadpool_info
    H = inp["H"]
    cu = inp["cu"].cpu().numpy()
    q = inp["q"].float().cpu().numpy().astype(np.float64)
    done_tok = 0.0
    pairs = 0
    t0 = time.perf_counter()
    b = 0
    while True:
        lo, hi = int(cu[b]), int(cu[b + 1])
        h = pairs % H
        kk = inp["k"][lo:hi, h].float().cpu().numpy().astype(np.float64)
        vv = inp["v"][lo:hi, h].float().cpu().numpy().astype(np.float64)
        ts = time.perf_counter()
        oracle.sa_problem(q[h], kk, vv, inp["scale"], 0)
        t_pair = time.perf_counter() - ts
        done_tok += (hi - lo) / H
        pairs += 1
        b = (b + 1) % inp["users"]
        if time.perf_counter() - t0 > budget_s or pairs >= 64:
            break
    elapsed_compute = time.perf_counter() - t0
    threads = 0
    for pool in threadpool_info():
        threads = max(threads, pool.get("num_threads", 0))
    return {"value": done_tok / elapsed_compute, "unit": UNIT, "cores": threads or os.cpu_count(),
            "kind": "oracle",
            "sample": f"{pairs} whole (user, head) problems of the workload, {done_tok:.0f} history-token "
                      f"equivalents (tokens x heads done / H), fp64 numpy, {elapsed_compute:.1f} s incl. "
                      f"host copies of the slices"}


def run_reference(args, rank, world):
    """--impl reference: the fp64 CPU oracle on the host cores, bounded samples per step."""
    if rank != 0:
        return
    import torch
    name = args.workload
    spec, H, d, kp, su = WORKLOADS[name]
    lens = lengths_for(spec, 0)
    rng = np.random.default_rng(2)
    q = (rng.standard_normal((H, kp, d), dtype=np.float32) / math.sqrt(d))
    q = torch.from_numpy(q).bfloat16().float().numpy().astype(np.float64)
    import oracle
    n = min(lens[0], 100_000)
    kk = torch.from_numpy(rng.standard_normal((n, d), dtype=np.float32)).bfloat16().float().numpy().astype(np.float64)
    vv = torch.from_numpy(rng.standard_normal((n, d), dtype=np.float32)).bfloat16().float().numpy().astype(np.float64)
    for _ in range(args.warmup if args.warmup < 1 else 1):
        oracle.sa_problem(q[0], kk[:1000], vv[:1000], 1.0, 0 if args.norm == "proto" else 1)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.sa_problem(q[0], kk, vv, 1.0, 0 if args.norm == "proto" else 1)
        times.append(time.perf_counter() - t0)
    tok_equiv = n / H
    ms = 1e3 * statistics.mean(times)
    value = tok_equiv / (ms / 1e3)
    from threadpoolctl import threadpool_info
    threads = max([p.get("num_threads", 0) for p in threadpool_info()] or [os.cpu_count()])
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": name, "norm": args.norm, "sample": f"one (user, head) problem of {n} tokens per step"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"one whole (user, head) problem ({n} tokens, k={kp}, d={d}) per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ska", choices=["ska", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--norm", default="proto", choices=["proto", "token"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU fallback)")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    from sketch_attention_flashsa_b200 import api, dp, flops

    inp = make_device_inputs(args.workload, rank, dev)
    H, d, kp, B = inp["H"], inp["d"], inp["k_protos"], inp["users"]
    T = inp["k"].shape[0]
    desc = api.sa_desc(inp["q"], inp["k"], inp["cu"], scale=inp["scale"], norm=args.norm)
    ws = torch.empty(api.sa_forward_workspace_size(desc), dtype=torch.uint8, device=dev)
    sketch = torch.empty((B, H, kp, d), dtype=torch.float32, device=dev)
    lse = torch.empty((T, H) if args.norm == "proto" else (B, H, kp), dtype=torch.float32, device=dev)

    def step():
        api.sa_forward(inp["q"], inp["k"], inp["v"], inp["cu"], inp["seqused"], scale=inp["scale"],
                       norm=args.norm, workspace=ws, out=sketch, lse_out=lse)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = api.read_device_status(ws)
    if st != 0:
        raise SystemExit(f"device status {st} after warm-up")

    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in kev:  # materialise the event handles
        a.record()
        b.record()
    torch.cuda.synchronize()
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        api.set_timing_events(*kev[i])
        step()
    e1.record()
    api.set_timing_events(None, None)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    ms_total = e0.elapsed_time(e1)
    kern_ms = [a.elapsed_time(b) for a, b in kev]
    ms_total, kern_mean = dp.max_over_ranks([ms_total, statistics.mean(kern_ms)], device=dev)
    ms_per_step = ms_total / args.steps
    valid = inp["valid"]
    total_tokens_all = valid * world
    value = total_tokens_all / (ms_per_step / 1e3)
    fl = flops.sa_forward_flops(valid, H, kp, d)
    by = flops.sa_forward_bytes(valid, H, kp, d, B, norm=0 if args.norm == "proto" else 1)
    tflops = fl / (ms_per_step / 1e3) / 1e12

    peaks = load_peaks()
    kname = "sa_proto_fwd_kernel" if args.norm == "proto" else "fa_fwd_kernel"
    t_tensor = fl / (peaks["bf16_tflops"] * 1e12)
    t_hbm = by / (peaks["hbm_gbs"] * 1e9)
    bound = "tensor" if t_tensor >= t_hbm else "hbm"
    if bound == "tensor":
        achieved = fl / (kern_mean / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "traffic": None,
                "peak_source": f"{peaks['source']} bf16 dense (burst); sustained {peaks['bf16_tflops_sustained']}",
                "kernel": kname, "kernel_ms": kern_mean}
    else:
        achieved = by / (kern_mean / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": None, "peak_source": peaks["source"],
                "kernel": kname, "kernel_ms": kern_mean}
    traffic_file = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(traffic_file):
        import hashlib
        with open(traffic_file) as f:
            tr = json.load(f).get(args.workload, {}).get(args.norm)
        if tr:
            with open(os.path.join(ROOT, tr["source"]), "rb") as f:
                cur = hashlib.sha256(f.read()).hexdigest()[:16]
            # counters are only valid for the kernel source they were taken on
            roof["traffic"] = tr["bytes"] if cur == tr["source_sha256"] else None

    # End to end through the public API: pinned host inputs -> device, forward, sketch -> host.
    hq = inp["q"].cpu().pin_memory()
    hk = inp["k"].cpu().pin_memory()
    hv = inp["v"].cpu().pin_memory()
    hcu = inp["cu"].cpu().pin_memory()
    hsu = inp["seqused"].cpu().pin_memory() if inp["seqused"] is not None else None
    hout = torch.empty(sketch.shape, dtype=torch.float32).pin_memory()
    dq, dk, dv, dcu = (torch.empty_like(x) for x in (inp["q"], inp["k"], inp["v"], inp["cu"]))
    dsu = torch.empty_like(inp["seqused"]) if hsu is not None else None

    def e2e_step():
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        dcu.copy_(hcu, non_blocking=True)
        if dsu is not None:
            dsu.copy_(hsu, non_blocking=True)
        api.sa_forward(dq, dk, dv, dcu, dsu, scale=inp["scale"], norm=args.norm, workspace=ws, out=sketch,
                       lse_out=lse)
        hout.copy_(sketch, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for _ in range(args.e2e_steps):
        e2e_step()
    f1.record()
    torch.cuda.synchronize()
    te = dp.max_over_ranks([f0.elapsed_time(f1) / args.e2e_steps], device=dev)
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hcu) + ((hsu,) if hsu is not None else ()))
    d2h = hout.numel() * hout.element_size()
    e2e = {"value": total_tokens_all / (float(te[0]) / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": float(te[0])}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(inp)

    launches_per_step = 3 + (1 if lse is not None else 0)
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": args.workload, "norm": args.norm, "users_per_gpu": B, "heads": H,
                           "head_dim": d, "protos": kp, "valid_tokens_per_gpu": valid,
                           "l2": "inputs larger than L2 (K and V are %.2f GB each per GPU)" % (
                               inp["k"].numel() * 2 / 1e9),
                           "parallelism": f"dp{world} (independent users per rank)"},
                "tflops": tflops, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches_per_step * args.steps, "clocks": clocks}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
