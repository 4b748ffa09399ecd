"""Seeded synthetic workloads for Sketch Attention (SA) and STCA.

This module is the only code shared by the CUDA path's tests, the bench and the
CPU oracle: it draws random inputs and nothing else. It contains none of the
method's arithmetic (no scores, no softmax, no aggregation).

The pages measure on proprietary Douyin histories (SequenceO1, §5 and App. G.5),
which are not available. The generators below stand in for them with the shapes
of those workloads: raw histories of up to n_max = 100K behaviours per user
(SequenceO1 §2.1), ragged across users, prototypes shared by every user
(SequenceO1 §3.1, Eq. (6)), and an STCA target batch per user that attends over
the recent 10K suffix and the user's sketch (SequenceO1 §3.4, §4.2).

Recipe (fixed, so that every consumer sees the same bits):

* ``rng = numpy.random.default_rng(seed)``.
* Draw order: (1) ragged lengths, if any; (2) Q; (3) K; (4) V; (5) extras
  (padding garbage, upstream gradients, sketch K/V for STCA).
* Ragged lengths: ``round(exp(U(ln 1000, ln 100000)))`` clipped to [1000, 100000].
* Normal draws are float32 ``standard_normal`` times a sigma; bf16 tensors are
  the round-to-nearest-even conversion of those float32 draws.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

NORM_PROTO = 0
NORM_TOKEN = 1


def ragged_lengths(rng: np.random.Generator, batch: int, lo: int = 1000,
                   hi: int = 100_000) -> np.ndarray:
    """Log-uniform history lengths in [lo, hi], the shape of a 100K-truncated feed."""
    x = np.exp(rng.uniform(math.log(lo), math.log(hi), batch))
    return np.clip(np.round(x), lo, hi).astype(np.int64)


def normal(rng: np.random.Generator, shape, sigma: float = 1.0) -> np.ndarray:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if sigma != 1.0:
        a *= np.float32(sigma)
    return a


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """Round-to-nearest-even float32 -> bfloat16 (host tensor)."""
    return torch.from_numpy(a).to(torch.bfloat16)


def cu_from_lengths(lengths) -> torch.Tensor:
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    assert cu[-1] < 2**31, "cu_seqlens must fit int32"
    return torch.from_numpy(cu.astype(np.int32))


@dataclasses.dataclass
class SAInputs:
    """One SA problem on the host.

    q: [H, k, d] (shared prototypes) or [B, H, k, d] (per-user queries)
    k, v: [total_tokens, H, d] packed by user
    cu_seqlens: int32 [B+1]; seqused: int32 [B] or None (valid prefix per user)
    """
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    cu_seqlens: torch.Tensor
    seqused: Optional[torch.Tensor]
    scale: float
    norm: int
    dsketch: Optional[torch.Tensor] = None

    @property
    def num_users(self) -> int:
        return int(self.cu_seqlens.numel() - 1)

    @property
    def num_heads(self) -> int:
        return int(self.k.shape[1])

    @property
    def head_dim(self) -> int:
        return int(self.k.shape[2])

    @property
    def num_protos(self) -> int:
        return int(self.q.shape[-2])

    @property
    def total_tokens(self) -> int:
        return int(self.k.shape[0])

    def valid_lengths(self) -> np.ndarray:
        cu = self.cu_seqlens.numpy().astype(np.int64)
        lens = cu[1:] - cu[:-1]
        if self.seqused is not None:
            lens = np.minimum(lens, self.seqused.numpy().astype(np.int64))
        return lens

    def valid_tokens(self) -> int:
        return int(self.valid_lengths().sum())


def make_sa(lengths, num_heads: int, head_dim: int, num_protos: int, seed: int,
            *, norm: int = NORM_PROTO, dtype: str = "bf16", q_sigma: Optional[float] = None,
            kv_sigma: float = 1.0, scale: float = 1.0, seqused=None,
            garbage_sigma: float = 100.0, per_user_q: bool = False,
            with_dsketch: bool = False, dsketch_seed: Optional[int] = None,
            ragged_batch: Optional[int] = None, length_fn=None) -> SAInputs:
    """Draw one SA workload.

    ``lengths``: list of per-user packed lengths, or None with ``ragged_batch``=B
    to draw log-uniform lengths first (step (1) of the recipe), or None with
    ``length_fn(rng)`` returning the lengths (also drawn first).
    ``seqused``: optional per-user valid prefix; rows past it are refilled with
    finite garbage N(0, garbage_sigma^2) in step (5).
    """
    rng = np.random.default_rng(seed)
    if lengths is None:
        lengths = length_fn(rng) if length_fn is not None else ragged_lengths(rng, ragged_batch)
    lengths = [int(x) for x in lengths]
    B, H, d, kp = len(lengths), num_heads, head_dim, num_protos
    total = int(sum(lengths))
    if q_sigma is None:
        q_sigma = 1.0 / math.sqrt(d)
    qshape = (B, H, kp, d) if per_user_q else (H, kp, d)
    q = normal(rng, qshape, q_sigma)
    k = normal(rng, (total, H, d), kv_sigma)
    v = normal(rng, (total, H, d), kv_sigma)
    su = None
    if seqused is not None:
        su_np = np.asarray(seqused, dtype=np.int64)
        cu = np.concatenate([[0], np.cumsum(lengths)])
        for b in range(B):
            lo, hi = cu[b] + min(su_np[b], lengths[b]), cu[b + 1]
            if hi > lo:
                k[lo:hi] = normal(rng, (hi - lo, H, d), garbage_sigma)
                v[lo:hi] = normal(rng, (hi - lo, H, d), garbage_sigma)
        su = torch.from_numpy(su_np.astype(np.int32))
    ds = None
    if with_dsketch:
        drng = rng if dsketch_seed is None else np.random.default_rng(dsketch_seed)
        ds = to_bf16(normal(drng, (B, H, kp, d)))
    if dtype == "bf16":
        qt, kt, vt = to_bf16(q), to_bf16(k), to_bf16(v)
    elif dtype == "f32":
        qt, kt, vt = torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v)
    else:
        raise ValueError(dtype)
    return SAInputs(qt, kt, vt, cu_from_lengths(lengths), su, float(scale), int(norm), ds)


@dataclasses.dataclass
class STCAInputs:
    """One STCA problem on the host.

    q: [total_targets, H, d]; cu_targets int32 [B+1]
    k_hist, v_hist: [total_hist, H, d]; cu_hist int32 [B+1]
    k_sk, v_sk: [B, H, ks, d] (may have ks == 0)
    target_kv_len: optional int32 [total_targets], per-target number of suffix keys
    """
    q: torch.Tensor
    cu_targets: torch.Tensor
    k_hist: torch.Tensor
    v_hist: torch.Tensor
    cu_hist: torch.Tensor
    k_sk: torch.Tensor
    v_sk: torch.Tensor
    scale: float
    target_kv_len: Optional[torch.Tensor] = None
    dout: Optional[torch.Tensor] = None  # bf16 [total_targets, H, d], the upstream gradient (backward)


def make_stca(targets, hist, num_heads: int, head_dim: int, num_sketch: int, seed: int,
              *, scale: Optional[float] = None, sigma: float = 1.0,
              with_kv_len: bool = False, with_dout: bool = False) -> STCAInputs:
    """Draw one STCA workload: per-user target counts ``targets`` and suffix lengths ``hist``."""
    rng = np.random.default_rng(seed)
    targets = [int(x) for x in targets]
    hist = [int(x) for x in hist]
    B, H, d = len(targets), num_heads, head_dim
    q = normal(rng, (sum(targets), H, d), sigma)
    kh = normal(rng, (sum(hist), H, d), sigma)
    vh = normal(rng, (sum(hist), H, d), sigma)
    ks = normal(rng, (B, H, num_sketch, d), sigma)
    vs = normal(rng, (B, H, num_sketch, d), sigma)
    kvl = None
    if with_kv_len:
        parts = [rng.integers(0, h + 1, size=t) for t, h in zip(targets, hist)]
        kvl = torch.from_numpy(np.concatenate(parts).astype(np.int32)) if parts else None
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dout = to_bf16(normal(rng, (sum(targets), H, d))) if with_dout else None
    return STCAInputs(to_bf16(q), cu_from_lengths(targets), to_bf16(kh), to_bf16(vh),
                      cu_from_lengths(hist), to_bf16(ks), to_bf16(vs), float(scale), kvl, dout)


# The five benchmark workloads plus the paper's production SA shape (App. G.5).

def config1() -> SAInputs:
    """1 user, L=1024, H=1, d=64, k=16; fp32 Q,K,V ~ N(0,1)/sqrt(d); seed 0."""
    s = 1.0 / math.sqrt(64)
    return make_sa([1024], 1, 64, 16, 0, dtype="f32", q_sigma=s, kv_sigma=s)


def config2(norm: int = NORM_PROTO) -> SAInputs:
    """64 ragged users in [1K, 100K], H=4, d=64, k=256 shared; seed 1."""
    return make_sa(None, 4, 64, 256, 1, norm=norm, ragged_batch=64)


def config3(norm: int = NORM_PROTO, masked: bool = False) -> SAInputs:
    """8 users x 100,000 tokens, H=8, d=128, k=512; seed 2.

    ``masked`` gives the padded variant: user 0 (10% of 8 users, rounded up)
    keeps its first 70,000 tokens and its last 30% hold finite garbage.
    """
    su = [70_000] + [100_000] * 7 if masked else None
    return make_sa([100_000] * 8, 8, 128, 512, 2, norm=norm, seqused=su)


def config4(norm: int = NORM_PROTO) -> SAInputs:
    """Backward at config-2 shapes; upstream dSketch bf16 N(0,1) drawn with seed 3."""
    return make_sa(None, 4, 64, 256, 1, norm=norm, ragged_batch=64, with_dsketch=True,
                   dsketch_seed=3)


def config5() -> STCAInputs:
    """STCA: 16 users x 512 targets, H=4, d=64, 10,000 suffix keys + 256 sketch keys; seed 4."""
    return make_stca([512] * 16, [10_000] * 16, 4, 64, 256, 4, scale=1.0 / 8.0)


def config_paper() -> SAInputs:
    """The paper's production SA shape: H=1, d=128, k=1024, 8 users, lengths ~ N(85K, 10K) <= 100K."""
    def lens(rng):
        return np.clip(np.round(rng.normal(85_000, 10_000, 8)), 1000, 100_000).astype(np.int64)
    return make_sa(None, 1, 128, 1024, 5, length_fn=lens)


@dataclasses.dataclass
class RefineInputs:
    """One refinement layer's inputs (SequenceO1 §3.3, Eq. (13)-(14)): [B, H, k, d] sketches and the
    per-head SwiGLU weights (App. G.1) and LayerNorm vectors."""
    x_tilde: torch.Tensor   # fp32 [B, H, k, d]
    x_hat: torch.Tensor     # fp32 [B, H, k, d]
    w1: torch.Tensor        # bf16 [H, d, F]
    wg: torch.Tensor        # bf16 [H, d, F]
    w2: torch.Tensor        # bf16 [H, F, d]
    gamma1: Optional[torch.Tensor] = None  # fp32 [H, d]
    beta1: Optional[torch.Tensor] = None
    gamma2: Optional[torch.Tensor] = None
    beta2: Optional[torch.Tensor] = None


def make_refine(B: int, H: int, k: int, d: int, seed: int, *, affine: bool = True,
                x_sigma: float = 1.0, hat_sigma: float = 1.0) -> RefineInputs:
    """Draw order: x_tilde, x_hat (N(0, sigma^2) fp32), W_1, W_g (N(0, 1/d)), W_2 (N(0, 1/F)), each
    rounded to bf16, F = 2d; with ``affine`` then gamma1, beta1, gamma2, beta2 as 1 + 0.1 N(0,1),
    0.1 N(0,1), 1 + 0.1 N(0,1), 0.1 N(0,1) in fp32."""
    rng = np.random.default_rng(seed)
    F = 2 * d
    xt = normal(rng, (B, H, k, d), x_sigma)
    xh = normal(rng, (B, H, k, d), hat_sigma)
    w1 = normal(rng, (H, d, F), 1.0 / math.sqrt(d))
    wg = normal(rng, (H, d, F), 1.0 / math.sqrt(d))
    w2 = normal(rng, (H, F, d), 1.0 / math.sqrt(F))
    out = RefineInputs(torch.from_numpy(xt), torch.from_numpy(xh), to_bf16(w1), to_bf16(wg), to_bf16(w2))
    if affine:
        out.gamma1 = torch.from_numpy(1.0 + normal(rng, (H, d), 0.1))
        out.beta1 = torch.from_numpy(normal(rng, (H, d), 0.1))
        out.gamma2 = torch.from_numpy(1.0 + normal(rng, (H, d), 0.1))
        out.beta2 = torch.from_numpy(normal(rng, (H, d), 0.1))
    return out


def config_refine() -> RefineInputs:
    """The refinement layer on the sketch of the 8 x 100K, H=8, d=128, k=512 workload; seed 6."""
    return make_refine(8, 8, 512, 128, 6)


@dataclasses.dataclass
class StackInputs:
    """N_sa stacked SA layers (SequenceO1 §3.3): prototypes, per-layer query weights and keys, the
    history X as values, and per-layer refinement parameters."""
    p0: torch.Tensor            # fp32 [H, k, d], P^(0)
    w_q: list                   # N_sa bf16 [H, d, d]
    keys: list                  # N_sa bf16 [T, H, d], K^(l) = X W_K^(l)
    v: torch.Tensor             # bf16 [T, H, d], X
    cu_seqlens: torch.Tensor    # int32 [B + 1]
    ffn: list                   # N_sa RefineInputs with only the weights and LN vectors set
    scale: float


def make_stack(lengths, num_heads: int, head_dim: int, num_protos: int, n_layers: int, seed: int) -> StackInputs:
    """Draw order: P^(0) (N(0, 1) fp32); the values X (N(0, 1), bf16); then per layer W_Q
    (N(0, 1/d), bf16), the keys (N(0, 1), bf16), W_1, W_g (N(0, 1/d)), W_2 (N(0, 1/F)) in bf16 and
    gamma1, beta1, gamma2, beta2 (1 + 0.1 N, 0.1 N, 1 + 0.1 N, 0.1 N; fp32). Scale 1/sqrt(d)."""
    rng = np.random.default_rng(seed)
    H, d, k = num_heads, head_dim, num_protos
    F = 2 * d
    T = int(sum(lengths))
    p0 = torch.from_numpy(normal(rng, (H, k, d)))
    v = to_bf16(normal(rng, (T, H, d)))
    w_q, keys, ffn = [], [], []
    for _ in range(n_layers):
        w_q.append(to_bf16(normal(rng, (H, d, d), 1.0 / math.sqrt(d))))
        keys.append(to_bf16(normal(rng, (T, H, d))))
        w1 = normal(rng, (H, d, F), 1.0 / math.sqrt(d))
        wg = normal(rng, (H, d, F), 1.0 / math.sqrt(d))
        w2 = normal(rng, (H, F, d), 1.0 / math.sqrt(F))
        r = RefineInputs(None, None, to_bf16(w1), to_bf16(wg), to_bf16(w2))
        r.gamma1 = torch.from_numpy(1.0 + normal(rng, (H, d), 0.1))
        r.beta1 = torch.from_numpy(normal(rng, (H, d), 0.1))
        r.gamma2 = torch.from_numpy(1.0 + normal(rng, (H, d), 0.1))
        r.beta2 = torch.from_numpy(normal(rng, (H, d), 0.1))
        ffn.append(r)
    return StackInputs(p0, w_q, keys, v, cu_from_lengths(lengths), ffn, 1.0 / math.sqrt(d))

