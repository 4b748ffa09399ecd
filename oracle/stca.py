"""fp64 oracle for STCA target-to-history cross-attention.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: SequenceO1 (arXiv 2609.08443), §2.3 "STCA Recap":
  Attn(q, X) = softmax((q W_Q)(X W_K)^T / sqrt(d_h)) (X W_V),
applied in §3.4 to the recent suffix (z_r = STCA_10k(x_t, X_r)) and to the
adapted sketch, with many targets of one user batched together by MRLB (§4.2).

Readings taken here: the projected query, keys and values are inputs; each
head is an independent attention; the keys of one target are the
concatenation [its user's suffix rows (optionally only the first
target_kv_len[t] of them) ; its user's sketch rows], under one softmax.
"""
from __future__ import annotations

import numpy as np


def _attend(q_t, keys, vals, scale):
    """One query row over a key set: returns (out [d], lse)."""
    if keys.shape[0] == 0:
        return np.zeros(vals.shape[1]), -np.inf
    s = scale * (keys @ q_t)                 # [n]
    m = s.max()
    lse = m + np.log(np.exp(s - m).sum())
    p = np.exp(s - lse)
    return p @ vals, lse


def stca_forward(q, cu_targets, k_hist, v_hist, cu_hist, k_sk, v_sk, scale,
                 target_kv_len=None):
    """Batched STCA forward.

    q [Tq,H,d]; k_hist, v_hist [Th,H,d]; k_sk, v_sk [B,H,ks,d] (ks may be 0).
    Returns out [Tq,H,d] and lse [Tq,H].
    """
    q = np.asarray(q, dtype=np.float64)
    kh = np.asarray(k_hist, dtype=np.float64)
    vh = np.asarray(v_hist, dtype=np.float64)
    ks = np.asarray(k_sk, dtype=np.float64)
    vs = np.asarray(v_sk, dtype=np.float64)
    cut = np.asarray(cu_targets, dtype=np.int64)
    cuh = np.asarray(cu_hist, dtype=np.int64)
    Tq, H, d = q.shape
    out = np.zeros((Tq, H, d))
    lse = np.full((Tq, H), -np.inf)
    for b in range(cut.shape[0] - 1):
        h_lo, h_hi = int(cuh[b]), int(cuh[b + 1])
        for t in range(int(cut[b]), int(cut[b + 1])):
            n_suffix = h_hi - h_lo
            if target_kv_len is not None:
                n_suffix = min(n_suffix, int(np.asarray(target_kv_len)[t]))
            for h in range(H):
                keys = np.concatenate([kh[h_lo:h_lo + n_suffix, h], ks[b, h]], axis=0)
                vals = np.concatenate([vh[h_lo:h_lo + n_suffix, h], vs[b, h]], axis=0)
                out[t, h], lse[t, h] = _attend(q[t, h], keys, vals, scale)
    return out, lse
