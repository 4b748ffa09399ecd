#!/usr/bin/env python
"""Benchmark of the Sketch Attention hot path on B200 (SequenceO1 §3.1 SA, §4.4 FlashSA, §2.3 STCA).

Default workload (the headline): the FlashSA forward on 8 users x 100,000 history tokens, H=8
heads, d=128, k=512 prototypes, prototype-wise normalisation (the paper's Eq. (8)), bf16 inputs,
fp32 sketch and per-token lse. One step = one sa_forward call (schedule, fused kernel, partial
combine, lse fill). The other rows of the path run with --workload (same JSON contract):

  sa_fwd_*                          one step = one sa_forward call (--norm proto|token)
  sa_bwd_b64_ragged_h4_d64_k256     one step = one sa_backward call: 64 ragged users (1.45M
                                    tokens), H=4, d=64, k=256 -> dQ, dK, dV (--norm proto|token)
  sa_bwd_b8_l100k_h8_d128_k512      the same at the headline shapes (launches over chunks of 128
                                    prototypes; the kernel time spans all of them)
  stca_b16_t512_h4_d64_l10k_s256    one step = one stca_forward call: 16 users x 512 targets over
                                    [10,000 suffix ; 256 sketch] keys, H=4, d=64

  python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--norm proto|token]
  python bench.py --impl reference ...   # the fp64 CPU oracle on a bounded sample

Multi-GPU (one process per GPU): `--gpus N` outside a launcher re-executes this script under
torch.distributed.run with N ranks. The global batch is N copies of the workload's users (ragged
lengths drawn for all N x B users at once); dp.partition_users assigns them to ranks balanced by
length, so each rank holds about one workload's worth (weak scaling) and computes its users with
no collective on the data path. The reported time is the max over ranks of the device-timed region.

The headline (default) line also carries the token-wise normalisation of the same workload on the
same inputs under "token", so that one run reports the forward in both normalisations.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
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

METRICS = {
    "sa_fwd": ("SA fwd history-tokens/s and TFLOP/s (fraction of B200 bf16 peak) at L=100K", "history-tokens/s"),
    "sa_bwd": ("SA bwd history-tokens/s (dQ, dK, dV with A recomputed) and TFLOP/s", "history-tokens/s"),
    "stca": ("STCA targets/s over [10K suffix ; 256 sketch] keys and TFLOP/s", "targets/s"),
    "refine": ("sketch refinement rows/s (LN, SwiGLU FFN, LN, next-layer query projection) and GB/s",
               "sketch-rows/s"),
    "sa_stack": ("stacked SA (N_sa = 2 layers) history-tokens/s at L=100K", "history-tokens/s"),
    "stca_bwd": ("STCA bwd targets/s (dq, dK, dV over [10K suffix ; 256 sketch] keys) and TFLOP/s", "targets/s"),
}

# name -> kind and shapes. lens: list, "ragged64" (64 users, log-uniform in [1K, 100K], seed 1) or
# "paper" (8 users, N(85K, 10K) clipped to [1K, 100K], seed 5).
WORKLOADS = {
    "sa_fwd_b8_l100k_h8_d128_k512": dict(kind="sa_fwd", lens=[100_000] * 8, H=8, d=128, k=512, seqused=None),
    "sa_fwd_b8_l100k_h8_d128_k512_masked": dict(kind="sa_fwd", lens=[100_000] * 8, H=8, d=128, k=512,
                                                seqused=[70_000] + [100_000] * 7),
    "sa_fwd_b64_ragged_h4_d64_k256": dict(kind="sa_fwd", lens="ragged64", H=4, d=64, k=256, seqused=None),
    # the paper's V = X (Eq. (9)): one tensor passed as both keys and values
    "sa_fwd_b8_l100k_h8_d128_k512_kv_alias": dict(kind="sa_fwd", lens=[100_000] * 8, H=8, d=128, k=512, seqused=None,
                                                  alias=True),
    "sa_fwd_paper_h1_d128_k1024": dict(kind="sa_fwd", lens="paper", H=1, d=128, k=1024, seqused=None),
    # profiling size: same per-tile work as the headline, 205 MB of K+V (> L2), ~0.25 ms
    "sa_fwd_b2_l100k_h2_d128_k512": dict(kind="sa_fwd", lens=[100_000] * 2, H=2, d=128, k=512, seqused=None),
    "sa_fwd_b2_l100k_h2_d128_k512_kv_alias": dict(kind="sa_fwd", lens=[100_000] * 2, H=2, d=128, k=512,
                                                  seqused=None, alias=True),
    "sa_bwd_b64_ragged_h4_d64_k256": dict(kind="sa_bwd", lens="ragged64", H=4, d=64, k=256, seqused=None),
    # profiling size for the backward: 2 x 100K, one head, same per-tile work
    "sa_bwd_b2_l100k_h1_d64_k256": dict(kind="sa_bwd", lens=[100_000] * 2, H=1, d=64, k=256, seqused=None),
    # the backward at the headline forward's shapes (k = 512, d = 128: four launches over chunks of 128
    # prototypes, PROTO with a delta pass per chunk first)
    "sa_bwd_b8_l100k_h8_d128_k512": dict(kind="sa_bwd", lens=[100_000] * 8, H=8, d=128, k=512, seqused=None),
    # profiling size for it: 2 x 100K, one head, the same per-tile work
    "sa_bwd_b2_l100k_h1_d128_k512": dict(kind="sa_bwd", lens=[100_000] * 2, H=1, d=128, k=512, seqused=None),
    # the refinement layer on the sketch of the 8 x 100K workload (8 users x 8 heads x 512 rows, d = 128)
    "refine_b8_h8_k512_d128": dict(kind="refine", B=8, H=8, k=512, d=128),
    # two stacked SA layers (§3.3) over the 8 x 100K workload, own keys per layer, V = the history
    "sa_stack2_b8_l100k_h8_d128_k512": dict(kind="sa_stack", lens=[100_000] * 8, H=8, d=128, k=512, layers=2),
    "stca_bwd_b16_t512_h4_d64_l10k_s256": dict(kind="stca_bwd", users=16, targets=512, hist=10_000, ks=256, H=4,
                                               d=64, scale=0.125),
    "stca_b16_t512_h4_d64_l10k_s256": dict(kind="stca", users=16, targets=512, hist=10_000, ks=256, H=4, d=64,
                                           scale=0.125),
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


def lengths_for(spec, copies=1):
    """Packed lengths of `copies` workloads' worth of users (one draw for all of them)."""
    if isinstance(spec, list):
        return spec * copies
    rng = np.random.default_rng(1 if spec == "ragged64" else 5)
    if spec == "ragged64":
        x = np.exp(rng.uniform(math.log(1000), math.log(100_000), 64 * copies))
        return [int(v) for v in np.clip(np.round(x), 1000, 100_000)]
    return [int(v) for v in np.clip(np.round(rng.normal(85_000, 10_000, 8 * copies)), 1000, 100_000)]


def rank_users(spec, rank, world):
    """This rank's users of the global batch (world copies of the workload), assigned by
    dp.partition_users (balanced by valid length): returns (lengths, seqused or None)."""
    from sketch_attention_flashsa_b200 import dp
    lens = lengths_for(spec["lens"], world)
    su = spec.get("seqused")
    su_all = (su * world) if su else None
    valid = [min(a, b) for a, b in zip(lens, su_all)] if su_all else lens
    mine = dp.partition_users(valid, world)[rank]
    return [lens[u] for u in mine], ([su_all[u] for u in mine] if su_all else None)


def oracle_threads():
    from threadpoolctl import threadpool_info
    return max([p.get("num_threads", 0) for p in threadpool_info()] or [0]) or os.cpu_count()


def f64(t):
    return t.float().cpu().numpy().astype(np.float64)


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


# ---------------------------------------------------------------------------------------- jobs
# A job draws its seeded synthetic inputs on the device, runs one step through the public API on a
# dict of device tensors (so that the end-to-end leg can run the same call on freshly copied
# inputs), and states the step's units, algorithmic FLOPs and bytes, and its fused kernel.

class SaFwdJob:
    def __init__(self, spec, norm, rank, world, dev, inputs=None):
        import torch
        from sketch_attention_flashsa_b200 import api, flops
        self.api, self.norm = api, norm
        lens, su = rank_users(spec, rank, world)
        H, d, kp = spec["H"], spec["d"], spec["k"]
        T, B = sum(lens), len(lens)
        if inputs is not None:
            self.inputs = inputs  # the same tensors as another job (the headline's token-wise line)
        else:
            gen = torch.Generator(device=dev)
            gen.manual_seed(1000 + rank)
            self.inputs = {
                "q": (torch.randn((H, kp, d), generator=gen, device=dev) / math.sqrt(d)).bfloat16(),
                "k": torch.randn((T, H, d), generator=gen, device=dev, dtype=torch.bfloat16),
                "cu": torch.tensor(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32), device=dev),
            }
            if not spec.get("alias"):
                self.inputs["v"] = torch.randn((T, H, d), generator=gen, device=dev, dtype=torch.bfloat16)
            if su:
                self.inputs["seqused"] = torch.tensor(np.array(su, dtype=np.int32), device=dev)
        self.valid = sum(min(a, b) for a, b in zip(lens, su)) if su else T
        self.B, self.H, self.d, self.kp = B, H, d, kp
        desc = api.sa_desc(self.inputs["q"], self.inputs["k"], self.inputs["cu"], scale=1.0, norm=norm)
        self.ws = torch.empty(api.sa_forward_workspace_size(desc), dtype=torch.uint8, device=dev)
        self.sketch = torch.empty((B, H, kp, d), dtype=torch.float32, device=dev)
        self.lse = torch.empty((T, H) if norm == "proto" else (B, H, kp), dtype=torch.float32, device=dev)
        self.units = self.valid
        self.flops = flops.sa_forward_flops(self.valid, H, kp, d)
        self.bytes = flops.sa_forward_bytes(self.valid, H, kp, d, B, norm=0 if norm == "proto" else 1,
                                            kv_alias=bool(spec.get("alias")))
        self.kernel = "sa_proto_fwd_kernel" if norm == "proto" else "fa_fwd_kernel"
        self.launches = 4 if norm == "proto" else 3
        self.config = {"users_per_gpu": B, "heads": H, "head_dim": d, "protos": kp, "norm": norm,
                       "valid_tokens_per_gpu": self.valid,
                       "l2": "inputs larger than L2 (K and V are %.2f GB each per GPU)" % (T * H * d * 2 / 1e9)}

    def run(self, x):
        v = x["v"] if "v" in x else x["k"]  # no "v": the values are the keys (V = X)
        self.api.sa_forward(x["q"], x["k"], v, x["cu"], x.get("seqused"), scale=1.0, norm=self.norm,
                            workspace=self.ws, out=self.sketch, lse_out=self.lse)
        return self.sketch

    def oracle_sample(self, budget_s):
        """Whole (user, head) problems of this workload through the oracle until about budget_s
        seconds; returns (history-token equivalents done, seconds, description)."""
        import oracle
        cu = self.inputs["cu"].cpu().numpy()
        q = f64(self.inputs["q"])
        done, pairs, b, t0 = 0.0, 0, 0, time.perf_counter()
        while time.perf_counter() - t0 < budget_s and pairs < 64:
            lo, hi = int(cu[b]), int(cu[b + 1])
            h = pairs % self.H
            vv = self.inputs.get("v", self.inputs["k"])
            oracle.sa_problem(q[h], f64(self.inputs["k"][lo:hi, h]), f64(vv[lo:hi, h]), 1.0,
                              0 if self.norm == "proto" else 1)
            done += (hi - lo) / self.H
            pairs += 1
            b = (b + 1) % self.B
        return done, time.perf_counter() - t0, f"{pairs} whole (user, head) problems, fp64 numpy"


class SaBwdJob:
    def __init__(self, spec, norm, rank, world, dev):
        import torch
        from sketch_attention_flashsa_b200 import api, flops
        self.api, self.norm = api, norm
        lens, _ = rank_users(spec, rank, world)
        H, d, kp = spec["H"], spec["d"], spec["k"]
        T, B = sum(lens), len(lens)
        gen = torch.Generator(device=dev)
        gen.manual_seed(2000 + rank)
        x = {
            "q": (torch.randn((H, kp, d), generator=gen, device=dev) / math.sqrt(d)).bfloat16(),
            "k": torch.randn((T, H, d), generator=gen, device=dev, dtype=torch.bfloat16),
            "v": torch.randn((T, H, d), generator=gen, device=dev, dtype=torch.bfloat16),
            "cu": torch.tensor(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32), device=dev),
            "dsketch": torch.randn((B, H, kp, d), generator=gen, device=dev, dtype=torch.bfloat16),
        }
        # the forward's saved statistics (and, token-wise, its sketch) are inputs of the backward
        sk, lse, _ = api.sa_forward(x["q"], x["k"], x["v"], x["cu"], None, scale=1.0, norm=norm)
        x["lse"] = lse
        if norm == "token":
            x["sketch"] = sk
        self.inputs = x
        self.valid, self.B, self.H, self.d, self.kp = T, B, H, d, kp
        self.outs = (torch.empty_like(x["q"], dtype=torch.float32), torch.empty_like(x["k"], dtype=torch.float32),
                     torch.empty_like(x["v"], dtype=torch.float32))
        desc = api.sa_desc(x["q"], x["k"], x["cu"], scale=1.0, norm=norm)
        self.ws = torch.empty(api.sa_backward_workspace_size(desc), dtype=torch.uint8, device=dev)
        self.units = T
        self.flops = flops.sa_backward_flops(T, H, kp, d)
        # K, V read (bf16), dK, dV written (fp32), saved statistics, dSketch (and sketch), Q and dQ
        self.bytes = (T * H * d * (2 + 2 + 4 + 4) + (T * H * 4 if norm == "proto" else B * H * kp * 4)
                      + B * H * kp * d * (2 + (4 if norm == "token" else 0)) + H * kp * d * (2 + 4))
        self.kernel = "sa_bwd_kernel"
        # schedule, then per chunk of prototypes the fused kernel, the dQ reduction and the padding
        # zeroing (PROTO over several chunks: one delta pass per chunk first)
        one = kp <= (256 if d == 64 else 128)
        nch = 1 if one else kp // (256 if d == 64 else 128)
        self.launches = 1 + 3 * nch + (nch if (norm == "proto" and nch > 1) else 0)
        self.chunks = nch
        self.config = {"users_per_gpu": B, "heads": H, "head_dim": d, "protos": kp, "norm": norm,
                       "tokens_per_gpu": T, "outputs": "dQ, dK, dV fp32", "prototype_chunks": nch,
                       "l2": "inputs larger than L2 (K and V are %.2f GB each per GPU)" % (T * H * d * 2 / 1e9)}

    def run(self, x):
        dq, _, _ = self.api.sa_backward(x["q"], x["k"], x["v"], x["cu"], None, x["lse"], x["dsketch"],
                                        x.get("sketch"), scale=1.0, norm=self.norm, workspace=self.ws,
                                        outs=self.outs)
        return dq

    def oracle_sample(self, budget_s):
        import oracle
        cu = self.inputs["cu"].cpu().numpy()
        q, do = f64(self.inputs["q"]), f64(self.inputs["dsketch"])
        nid = 0 if self.norm == "proto" else 1
        done, users, t0 = 0.0, 0, time.perf_counter()
        order = np.argsort(np.diff(cu))  # shortest users first, so that the sample stays bounded
        for b in order:
            if time.perf_counter() - t0 > budget_s or users >= 16:
                break
            lo, hi = int(cu[b]), int(cu[b + 1])
            oracle.sa_backward(q, f64(self.inputs["k"][lo:hi]), f64(self.inputs["v"][lo:hi]), np.array([0, hi - lo]),
                               None, do[b:b + 1], 1.0, nid)
            done += hi - lo
            users += 1
        return done, time.perf_counter() - t0, f"{users} whole users (all heads, dQ dK dV), fp64 numpy"


class StcaJob:
    def __init__(self, spec, norm, rank, world, dev):
        import torch
        from sketch_attention_flashsa_b200 import api, flops
        self.api = api
        B, Tq, L, ks, H, d = spec["users"], spec["targets"], spec["hist"], spec["ks"], spec["H"], spec["d"]
        gen = torch.Generator(device=dev)
        gen.manual_seed(3000 + rank)
        x = {
            "q": torch.randn((B * Tq, H, d), generator=gen, device=dev, dtype=torch.bfloat16),
            "cu_t": torch.arange(0, B * Tq + 1, Tq, dtype=torch.int32, device=dev),
            "k_hist": torch.randn((B * L, H, d), generator=gen, device=dev, dtype=torch.bfloat16),
            "v_hist": torch.randn((B * L, H, d), generator=gen, device=dev, dtype=torch.bfloat16),
            "cu_h": torch.arange(0, B * L + 1, L, dtype=torch.int32, device=dev),
            "k_sk": torch.randn((B, H, ks, d), generator=gen, device=dev, dtype=torch.bfloat16),
            "v_sk": torch.randn((B, H, ks, d), generator=gen, device=dev, dtype=torch.bfloat16),
        }
        self.inputs, self.scale, self.Tq, self.B, self.H = x, spec["scale"], Tq, B, H
        self.out = torch.empty((B * Tq, H, d), dtype=torch.float32, device=dev)
        self.lse = torch.empty((B * Tq, H), dtype=torch.float32, device=dev)
        desc = api.stca_desc(x["q"], x["k_hist"], x["k_sk"], x["cu_t"], x["cu_h"], scale=self.scale, max_targets=Tq)
        self.ws = torch.empty(max(api.stca_forward_workspace_size(desc), 256), dtype=torch.uint8, device=dev)
        self.units = B * Tq
        self.flops = flops.stca_forward_flops(B * Tq, L + ks, H, d)
        self.bytes = B * Tq * H * d * (2 + 4) + B * Tq * H * 4 + 2 * B * L * H * d * 2 + 2 * B * H * ks * d * 2
        self.kernel = "fa_fwd_kernel"
        self.launches = 3
        self.config = {"users_per_gpu": B, "targets_per_user": Tq, "suffix_keys": L, "sketch_keys": ks, "heads": H,
                       "head_dim": d, "scale": self.scale,
                       "l2": "inputs larger than L2 (suffix K and V are %.0f MB together per GPU)" % (
                           2 * B * L * H * d * 2 / 1e6)}

    def run(self, x):
        out, _ = self.api.stca_forward(x["q"], x["cu_t"], x["k_hist"], x["v_hist"], x["cu_h"], x["k_sk"], x["v_sk"],
                                       scale=self.scale, max_targets=self.Tq, workspace=self.ws, out=self.out,
                                       lse_out=self.lse)
        return out

    def oracle_sample(self, budget_s):
        import oracle
        x = self.inputs
        cut, cuh = x["cu_t"].cpu().numpy(), x["cu_h"].cpu().numpy()
        done, users, t0 = 0.0, 0, time.perf_counter()
        per_user = 64
        while time.perf_counter() - t0 < budget_s and users < self.B:
            b = users
            rows = slice(int(cut[b]), int(cut[b]) + per_user)
            oracle.stca_forward(f64(x["q"][rows]), np.array([0, per_user]), f64(x["k_hist"][cuh[b]:cuh[b + 1]]),
                                f64(x["v_hist"][cuh[b]:cuh[b + 1]]), np.array([0, cuh[b + 1] - cuh[b]]),
                                f64(x["k_sk"][b:b + 1]), f64(x["v_sk"][b:b + 1]), self.scale, None)
            done += per_user
            users += 1
        return done, time.perf_counter() - t0, f"{per_user} targets of each of {users} users (all heads), fp64 numpy"


class RefineJob:
    """One refinement layer (residual + LN, SwiGLU FFN, residual + LN, the next layer's queries) on
    every sketch row. Its inputs (59 MB a set) fit in L2, so the steps rotate over four sets of
    inputs and outputs (236 MB together): a step's data were last touched three steps earlier."""
    SETS = 4

    def __init__(self, spec, norm, rank, world, dev):
        import torch
        from sketch_attention_flashsa_b200 import api, flops
        self.api = api
        B, H, k, d = spec["B"], spec["H"], spec["k"], spec["d"]
        F = 2 * d
        gen = torch.Generator(device=dev)
        gen.manual_seed(4000 + rank)
        rn = lambda *shape: torch.randn(shape, generator=gen, device=dev)  # noqa: E731
        self.weights = {"w1": (rn(H, d, F) / math.sqrt(d)).bfloat16(), "wg": (rn(H, d, F) / math.sqrt(d)).bfloat16(),
                        "w2": (rn(H, F, d) / math.sqrt(F)).bfloat16(), "wq": (rn(H, d, d) / math.sqrt(d)).bfloat16(),
                        "g1": 1 + rn(H, d) / 10, "b1": rn(H, d) / 10, "g2": 1 + rn(H, d) / 10, "b2": rn(H, d) / 10}
        self.sets = [{"x_tilde": rn(B, H, k, d), "x_hat": rn(B, H, k, d)} for _ in range(self.SETS)]
        self.outs = [torch.empty((B, H, k, d), device=dev) for _ in range(self.SETS)]
        self.inputs = self.sets[0]
        self.turn = 0
        self.ws = torch.empty(256, dtype=torch.uint8, device=dev)
        rows = B * H * k
        self.units = rows
        self.flops = flops.refine_flops(rows, d)
        self.bytes = flops.refine_bytes(rows, H, d)
        self.kernel = "sa_refine_kernel"
        self.launches = 2
        self.config = {"users_per_gpu": B, "heads": H, "rows_per_user_head": k, "head_dim": d, "ffn_dim": F,
                       "outputs": "x_next fp32, q_next bf16",
                       "l2": f"rotating over {self.SETS} input/output sets of {rows * d * 14 / 1e6:.0f} MB each"}

    def run(self, x):
        if x is self.inputs:  # the timed steps rotate over the sets
            i = self.turn % self.SETS
            self.turn += 1
            x, out = self.sets[i], self.outs[i]
        else:
            out = self.outs[0]
        w = self.weights
        x_next, _, _, q_next = self.api.sa_refine(x["x_tilde"], x["x_hat"], w["w1"], w["wg"], w["w2"], w["g1"],
                                                  w["b1"], w["g2"], w["b2"], w_q_next=w["wq"], workspace=self.ws,
                                                  out=out)
        return x_next

    def oracle_sample(self, budget_s):
        import oracle
        x, w = self.inputs, {n: f64(t) for n, t in self.weights.items()}
        B = x["x_tilde"].shape[0]
        done, users, t0 = 0.0, 0, time.perf_counter()
        while time.perf_counter() - t0 < budget_s and users < 64:
            b = users % B
            xt, xh = f64(x["x_tilde"][b:b + 1]), f64(x["x_hat"][b:b + 1])
            _, xn = oracle.refine(xt, xh, w["w1"], w["wg"], w["w2"], w["g1"], w["b1"], w["g2"], w["b2"])
            oracle.project_queries(xn, w["wq"])
            done += xt.shape[1] * xt.shape[2]
            users += 1
        return done, time.perf_counter() - t0, f"{users} whole users (all heads and rows), fp64 numpy"


class StackJob:
    """N_sa stacked SA layers (§3.3) through the public API: the layer-0 queries P^(0) W_Q, then per
    layer the prototype-wise SA forward over that layer's keys with V = the history, and the
    refinement that also emits the next layer's queries. The roofline is taken over the whole step
    (several kernels), against the bf16 tensor peak."""

    def __init__(self, spec, norm, rank, world, dev):
        import torch
        from sketch_attention_flashsa_b200 import api, flops
        self.api = api
        lens, _ = rank_users(spec, rank, world)
        H, d, kp, nl = spec["H"], spec["d"], spec["k"], spec["layers"]
        T, B = sum(lens), len(lens)
        F = 2 * d
        gen = torch.Generator(device=dev)
        gen.manual_seed(5000 + rank)
        rn = lambda *shape: torch.randn(shape, generator=gen, device=dev)  # noqa: E731
        x = {"p0": rn(H, kp, d), "v": rn(T, H, d).bfloat16(),
             "cu": torch.tensor(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32), device=dev)}
        for l in range(nl):
            x[f"k{l}"] = rn(T, H, d).bfloat16()
            x[f"wq{l}"] = (rn(H, d, d) / math.sqrt(d)).bfloat16()
            x[f"w1_{l}"] = (rn(H, d, F) / math.sqrt(d)).bfloat16()
            x[f"wg_{l}"] = (rn(H, d, F) / math.sqrt(d)).bfloat16()
            x[f"w2_{l}"] = (rn(H, F, d) / math.sqrt(F)).bfloat16()
        self.inputs, self.nl, self.scale = x, nl, 1.0 / math.sqrt(d)
        need = 0
        for qshape in ((H, kp, d), (B, H, kp, d)):  # layer 0 shares its queries, later layers do not
            q = torch.empty(qshape, dtype=torch.bfloat16, device=dev)
            need = max(need, api.sa_forward_workspace_size(api.sa_desc(q, x["v"], x["cu"], scale=self.scale,
                                                                         norm="proto")))
        self.ws = torch.empty(need, dtype=torch.uint8, device=dev)
        rows = B * H * kp
        self.units = T
        self.flops = nl * (flops.sa_forward_flops(T, H, kp, d) + flops.refine_flops(rows, d)) + flops.gemm(H * kp, d, d)
        self.bytes = nl * (flops.sa_forward_bytes(T, H, kp, d, B, norm=0) + flops.refine_bytes(rows, H, d))
        self.kernel = "step: sa_proto_fwd_kernel x2, sa_refine_kernel x3 (one projection-only) and small kernels"
        self.launches = 1 + nl * 6
        self.hook = False
        self.config = {"users_per_gpu": B, "heads": H, "head_dim": d, "protos": kp, "layers": nl, "norm": "proto",
                       "valid_tokens_per_gpu": T, "keys": "one key tensor per layer; values = the history",
                       "l2": "inputs larger than L2 (each K and V is %.2f GB per GPU)" % (T * H * d * 2 / 1e9)}

    def run(self, x):
        api = self.api
        q = api.project_queries(x["p0"], x["wq0"])
        x_t = x["p0"]
        for l in range(self.nl):
            sk, _, _ = api.sa_forward(q, x[f"k{l}"], x["v"], x["cu"], None, scale=self.scale, norm="proto",
                                      want_lse=False, workspace=self.ws)
            wq = x.get(f"wq{l + 1}")
            x_t, _, _, q = api.sa_refine(x_t, sk, x[f"w1_{l}"], x[f"wg_{l}"], x[f"w2_{l}"], w_q_next=wq)
        return x_t

    def oracle_sample(self, budget_s):
        import oracle
        x = self.inputs
        cu = x["cu"].cpu().numpy()
        t0 = time.perf_counter()
        n = min(2000, int(cu[1]))  # the first 2000 tokens of user 0, all heads, both layers
        sub = lambda t: f64(t[:n])  # noqa: E731
        ffn = [(f64(x[f"w1_{l}"]), f64(x[f"wg_{l}"]), f64(x[f"w2_{l}"]), None, None, None, None)
               for l in range(self.nl)]
        oracle.stacked_sa(f64(x["p0"]), [f64(x[f"wq{l}"]) for l in range(self.nl)],
                          [sub(x[f"k{l}"]) for l in range(self.nl)], sub(x["v"]), np.array([0, n]), None,
                          self.scale, ffn)
        return n, time.perf_counter() - t0, f"the first {n} tokens of one user through {self.nl} layers, fp64 numpy"


class StcaBwdJob(StcaJob):
    """The STCA backward at the forward's shapes: the forward's out and lse are computed once
    (inputs of the step), the upstream gradient is drawn; a step is one stca_backward call (its
    key-major and query-major kernels are timed together)."""

    def __init__(self, spec, norm, rank, world, dev):
        import torch
        from sketch_attention_flashsa_b200 import flops
        super().__init__(spec, norm, rank, world, dev)
        x = self.inputs
        gen = torch.Generator(device=dev)
        gen.manual_seed(3500 + rank)
        x["dout"] = torch.randn(x["q"].shape, generator=gen, device=dev, dtype=torch.bfloat16)
        out, lse = self.api.stca_forward(x["q"], x["cu_t"], x["k_hist"], x["v_hist"], x["cu_h"], x["k_sk"], x["v_sk"],
                                         scale=self.scale, max_targets=self.Tq)
        x["out"], x["lse"] = out, lse
        B, Tq, L, ks, H, d = spec["users"], spec["targets"], spec["hist"], spec["ks"], spec["H"], spec["d"]
        desc = self.api.stca_desc(x["q"], x["k_hist"], x["k_sk"], x["cu_t"], x["cu_h"], scale=self.scale,
                                  max_targets=Tq)
        self.ws = torch.empty(max(int(self.api._lib.lib().stca_backward_workspace_size(
            __import__("ctypes").byref(desc))), 256), dtype=torch.uint8, device=dev)
        # five GEMM-shaped products per (target, key): S, dP, dV, dK, dq (App. G.1 counting)
        self.flops = 2.5 * flops.stca_forward_flops(B * Tq, L + ks, H, d)
        # read q, dO (bf16), out (fp32), K and V (bf16), lse; write dq, dK, dV (fp32)
        self.bytes = (B * Tq * H * d * (2 + 2 + 4 + 4) + B * Tq * H * 4 + 2 * B * L * H * d * (2 + 4)
                      + 2 * B * H * ks * d * (2 + 4))
        self.kernel = "stca_bwd_dkv_kernel + stca_bwd_dq_kernel"
        self.launches = 5
        self.config["outputs"] = "dq, dK, dV fp32"

    def run(self, x):
        g = self.api.stca_backward(x["q"], x["cu_t"], x["k_hist"], x["v_hist"], x["cu_h"], x["k_sk"], x["v_sk"],
                                   x["out"], x["lse"], x["dout"], scale=self.scale, workspace=self.ws)
        return g[0]

    def oracle_sample(self, budget_s):
        import oracle
        x = self.inputs
        cut, cuh = x["cu_t"].cpu().numpy(), x["cu_h"].cpu().numpy()
        done, users, t0 = 0.0, 0, time.perf_counter()
        per_user = 16
        while time.perf_counter() - t0 < budget_s and users < self.B:
            b = users
            rows = slice(int(cut[b]), int(cut[b]) + per_user)
            oracle.stca_backward(f64(x["q"][rows]), np.array([0, per_user]), f64(x["k_hist"][cuh[b]:cuh[b + 1]]),
                                 f64(x["v_hist"][cuh[b]:cuh[b + 1]]), np.array([0, cuh[b + 1] - cuh[b]]),
                                 f64(x["k_sk"][b:b + 1]), f64(x["v_sk"][b:b + 1]), self.scale,
                                 f64(x["dout"][rows]), None)
            done += per_user
            users += 1
        return done, time.perf_counter() - t0, f"{per_user} targets of each of {users} users (all heads), fp64 numpy"


JOBS = {"sa_fwd": SaFwdJob, "sa_bwd": SaBwdJob, "stca": StcaJob, "refine": RefineJob, "sa_stack": StackJob,
        "stca_bwd": StcaBwdJob}


def traffic_for(workload, norm):
    """DRAM bytes per launch of the fused kernel from a committed ncu capture, or None when the
    kernel source has changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        tr = json.load(f).get(workload, {}).get(norm)
    if not tr:
        return None
    with open(os.path.join(ROOT, tr["source"]), "rb") as f:
        cur = hashlib.sha256(f.read()).hexdigest()[:16]
    return tr["bytes"] if cur == tr["source_sha256"] else None


def run_reference(args, rank, world):
    """--impl reference: the fp64 CPU oracle on the host cores, a bounded sample per step."""
    if rank != 0:
        return
    spec = WORKLOADS[args.workload]
    metric, unit = METRICS[spec["kind"]]
    job = _host_job(spec, args.norm)
    budget = args.ref_seconds if args.ref_seconds is not None else (4.0 if args.steps > 5 else 10.0)
    job.oracle_sample(0.01)  # warm-up: imports and first calls
    times, units, desc = [], [], ""
    for _ in range(args.steps):
        u, t, desc = job.oracle_sample(budget)
        times.append(t)
        units.append(u)
    value = sum(units) / sum(times)
    ms = 1e3 * statistics.mean(times)
    cores = oracle_threads()
    line = {"impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "norm": args.norm, "sample": desc},
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                             "sample": f"per step: {desc}, about {budget:.0f} s"},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _host_job(spec, norm):
    """A job's inputs drawn on the host, the same distributions, for the oracle alone (the
    reference arm touches neither the GPU nor libska.so)."""
    import types
    import torch
    g = torch.Generator().manual_seed(7)
    job = types.SimpleNamespace()
    rn = lambda *shape: torch.randn(shape, generator=g)  # noqa: E731
    if spec["kind"] == "refine":
        H, k, d = spec["H"], spec["k"], spec["d"]
        F = 2 * d
        job.inputs = {"x_tilde": rn(2, H, k, d), "x_hat": rn(2, H, k, d)}
        job.weights = {"w1": (rn(H, d, F) / math.sqrt(d)).bfloat16(), "wg": (rn(H, d, F) / math.sqrt(d)).bfloat16(),
                       "w2": (rn(H, F, d) / math.sqrt(F)).bfloat16(), "wq": (rn(H, d, d) / math.sqrt(d)).bfloat16(),
                       "g1": 1 + rn(H, d) / 10, "b1": rn(H, d) / 10, "g2": 1 + rn(H, d) / 10, "b2": rn(H, d) / 10}
        job.oracle_sample = types.MethodType(RefineJob.oracle_sample, job)
        return job
    if spec["kind"] == "sa_stack":
        H, kp, d, nl = spec["H"], spec["k"], spec["d"], spec["layers"]
        F, T = 2 * d, 2000
        x = {"p0": rn(H, kp, d), "v": rn(T, H, d).bfloat16(), "cu": torch.tensor([0, T], dtype=torch.int32)}
        for l in range(nl):
            x[f"k{l}"] = rn(T, H, d).bfloat16()
            x[f"wq{l}"] = (rn(H, d, d) / math.sqrt(d)).bfloat16()
            x[f"w1_{l}"] = (rn(H, d, F) / math.sqrt(d)).bfloat16()
            x[f"wg_{l}"] = (rn(H, d, F) / math.sqrt(d)).bfloat16()
            x[f"w2_{l}"] = (rn(H, F, d) / math.sqrt(F)).bfloat16()
        job.inputs, job.nl, job.scale = x, nl, 1.0 / math.sqrt(d)
        job.oracle_sample = types.MethodType(StackJob.oracle_sample, job)
        return job
    if spec["kind"] in ("stca", "stca_bwd"):
        B, Tq, L, ks, H, d = 2, 64, spec["hist"], spec["ks"], spec["H"], spec["d"]
        job.inputs = {"q": torch.randn((B * Tq, H, d), generator=g).bfloat16(),
                      "cu_t": torch.arange(0, B * Tq + 1, Tq, dtype=torch.int32),
                      "k_hist": torch.randn((B * L, H, d), generator=g).bfloat16(),
                      "v_hist": torch.randn((B * L, H, d), generator=g).bfloat16(),
                      "cu_h": torch.arange(0, B * L + 1, L, dtype=torch.int32),
                      "k_sk": torch.randn((B, H, ks, d), generator=g).bfloat16(),
                      "v_sk": torch.randn((B, H, ks, d), generator=g).bfloat16()}
        job.scale, job.B = spec["scale"], B
        if spec["kind"] == "stca_bwd":
            job.inputs["dout"] = torch.randn((B * Tq, H, d), generator=g).bfloat16()
        job.oracle_sample = types.MethodType((StcaBwdJob if spec["kind"] == "stca_bwd" else StcaJob).oracle_sample,
                                             job)
        return job
    lens = lengths_for(spec["lens"])
    H, d, kp = spec["H"], spec["d"], spec["k"]
    # a bounded sample: the shortest users of the workload, up to 4 of them
    take = sorted(lens)[:4]
    T = sum(take)
    job.inputs = {"q": (torch.randn((H, kp, d), generator=g) / math.sqrt(d)).bfloat16(),
                  "k": torch.randn((T, H, d), generator=g).bfloat16(), "v": torch.randn((T, H, d), generator=g).bfloat16(),
                  "cu": torch.tensor(np.concatenate([[0], np.cumsum(take)]).astype(np.int32)),
                  "dsketch": torch.randn((len(take), H, kp, d), generator=g).bfloat16()}
    job.norm, job.H, job.B = norm, H, len(take)
    cls = SaFwdJob if spec["kind"] == "sa_fwd" else SaBwdJob
    job.oracle_sample = types.MethodType(cls.oracle_sample, job)
    return job


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
    ap.add_argument("--no-token", action="store_true", help="headline: skip the token-wise line")
    ap.add_argument("--ref-seconds", type=float, default=None,
                    help="--impl reference: seconds of oracle work per step (default 4, or 10 for <= 5 steps)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # not under a launcher: start one process per GPU and pass this run's exit status through
        sys.exit(subprocess.call(launcher_command(args.gpus, sys.argv[1:])))
    if "WORLD_SIZE" in os.environ and world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")

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

    from sketch_attention_flashsa_b200 import api, dp

    spec = WORKLOADS[args.workload]
    metric, unit = METRICS[spec["kind"]]
    job = JOBS[spec["kind"]](spec, args.norm, rank, world, dev)
    peaks = load_peaks()
    res = time_job(job, args, world, dev, peaks)
    res["roofline"]["traffic"] = traffic_for(args.workload, {"stca": "stca", "refine": "refine",
                                                             "stca_bwd": "stca_bwd"}.get(spec["kind"], args.norm))

    # End to end through the public API: pinned host inputs -> device, the call, result -> host.
    host = {n: t.cpu().pin_memory() for n, t in job.inputs.items()}
    devx = {n: torch.empty_like(t) for n, t in job.inputs.items()}
    out = job.run(job.inputs)
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    def e2e_step():
        for n in host:
            devx[n].copy_(host[n], non_blocking=True)
        r = job.run(devx)
        hout.copy_(r, non_blocking=True)

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
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = hout.numel() * hout.element_size()
    e2e = {"value": res["units_all"] / (te[0] / 1e3), "unit": unit, "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": te[0], "result_read_back": list(hout.shape)}
    del host, devx

    # The headline also reports the token-wise normalisation on the same inputs.
    token = None
    if spec["kind"] == "sa_fwd" and args.norm == "proto" and not args.no_token:
        tjob = SaFwdJob(spec, "token", rank, world, dev, inputs=job.inputs)
        tres = time_job(tjob, args, world, dev, peaks)
        tres["roofline"]["traffic"] = traffic_for(args.workload, "token")
        token = {"value": tres["value"], "unit": unit, "ms_per_step": tres["ms_per_step"], "tflops": tres["tflops"],
                 "roofline": tres["roofline"], "gpu_launches": tjob.launches * args.steps, "clocks": tres["clocks"]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        done, secs, desc = job.oracle_sample(12.0)
        cpu = {"value": done / secs, "unit": unit, "cores": oracle_threads(), "kind": "oracle",
               "sample": f"{desc}, {secs:.1f} s incl. host copies of the slices"}

    if rank == 0:
        line = {"metric": metric, "value": res["value"], "unit": unit, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": args.workload, **job.config,
                           "parallelism": f"dp{world} (users partitioned over ranks by length, no collective)"},
                "tflops": res["tflops"], "roofline": res["roofline"], "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": job.launches * args.steps, "clocks": res["clocks"]}
        if token is not None:
            line["token"] = token
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def launcher_command(gpus, argv):
    """torch.distributed.run with one process per GPU on this node (rendezvous on 127.0.0.1)."""
    import socket
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
            "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]


def time_job(job, args, world, dev, peaks):
    """W warm-up steps, then K steps between a barrier and a synchronize on both sides, timed with
    CUDA events on the launching stream (the whole step and, through the library's timing hook,
    its fused kernel); clocks sampled meanwhile; times are the max over ranks."""
    import torch
    import torch.distributed as dist
    from sketch_attention_flashsa_b200 import api, dp

    for _ in range(args.warmup):
        job.run(job.inputs)
    torch.cuda.synchronize()
    st = api.read_device_status(job.ws)
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
    hook = getattr(job, "hook", True)  # False: several kernels a step, the step is the unit timed
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        if hook:
            api.set_timing_events(*kev[i])
        job.run(job.inputs)
    e1.record()
    api.set_timing_events(None, None)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    kern_mean = statistics.mean(a.elapsed_time(b) for a, b in kev) if hook else e0.elapsed_time(e1) / args.steps
    ms_total, kern_max = dp.max_over_ranks([e0.elapsed_time(e1), kern_mean], device=dev)
    units_all, flops_all = dp.sum_over_ranks([job.units, job.flops], device=dev)
    ms_per_step = ms_total / args.steps
    t_tensor = job.flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = job.bytes / (peaks["hbm_gbs"] * 1e9)
    # the dominant kernel's rate on each rank (its own work over its own kernel time), slowest rank
    if t_tensor >= t_hbm:
        achieved = -dp.max_over_ranks([-(job.flops / (kern_mean / 1e3) / 1e12)], device=dev)[0]
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "traffic": None,
                "peak_source": f"{peaks['source']} bf16 dense (burst); sustained {peaks['bf16_tflops_sustained']}"}
    else:
        achieved = -dp.max_over_ranks([-(job.bytes / (kern_mean / 1e3) / 1e9)], device=dev)[0]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": None, "peak_source": peaks["source"]}
    roof.update({"kernel": job.kernel, "kernel_ms": kern_max, "algorithmic_flops": job.flops,
                 "algorithmic_bytes": job.bytes})
    return {"ms_per_step": ms_per_step, "value": units_all / (ms_per_step / 1e3),
            "tflops": flops_all / (ms_per_step / 1e3) / 1e12, "roofline": roof, "clocks": clocks,
            "units_all": units_all}


if __name__ == "__main__":
    main()
