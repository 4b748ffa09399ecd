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


def stca_backward(q, cu_targets, k_hist, v_hist, cu_hist, k_sk, v_sk, scale, dout, target_kv_len=None):
    """Gradients of <dO, out> for the batched STCA forward above (STCA is trained end to end with
    the ranker, §2.3 and §3.4; its sketch branch passes gradients back into the sketch).

    For one target t, head h with keys K_t (its suffix rows, then its user's sketch rows), values
    V_t, p = softmax(scale K_t q_t) and out_t = p V_t:
      dV_t = p dO_t^T (per key row),  dp = V_t dO_t,  ds = p * (dp - <dO_t, out_t>),
      dq_t = scale ds K_t,  dK_t = scale ds q_t^T.
    Gradients of keys and values shared by several targets of a user are summed over them.
    Returns dq [Tq,H,d], dk_hist, dv_hist [Th,H,d], dk_sk, dv_sk [B,H,ks,d].
    """
    q = np.asarray(q, dtype=np.float64)
    kh = np.asarray(k_hist, dtype=np.float64)
    vh = np.asarray(v_hist, dtype=np.float64)
    ks = np.asarray(k_sk, dtype=np.float64)
    vs = np.asarray(v_sk, dtype=np.float64)
    do = np.asarray(dout, dtype=np.float64)
    cut = np.asarray(cu_targets, dtype=np.int64)
    cuh = np.asarray(cu_hist, dtype=np.int64)
    Tq, H, d = q.shape
    nsk = ks.shape[2]
    dq = np.zeros_like(q)
    dkh, dvh = np.zeros_like(kh), np.zeros_like(vh)
    dks, dvs = np.zeros_like(ks), np.zeros_like(vs)
    for b in range(cut.shape[0] - 1):
        h_lo, h_hi = int(cuh[b]), int(cuh[b + 1])
        for t in range(int(cut[b]), int(cut[b + 1])):
            n_suffix = h_hi - h_lo
            if target_kv_len is not None:
                n_suffix = min(n_suffix, int(np.asarray(target_kv_len)[t]))
            for h in range(H):
                keys = np.concatenate([kh[h_lo:h_lo + n_suffix, h], ks[b, h]], axis=0)
                vals = np.concatenate([vh[h_lo:h_lo + n_suffix, h], vs[b, h]], axis=0)
                if keys.shape[0] == 0:
                    continue
                s = scale * (keys @ q[t, h])
                pr = np.exp(s - s.max())
                pr /= pr.sum()
                out_t = pr @ vals
                dvals = np.outer(pr, do[t, h])
                dp = vals @ do[t, h]
                ds = pr * (dp - do[t, h] @ out_t)
                dq[t, h] = scale * (ds @ keys)
                dkeys = scale * np.outer(ds, q[t, h])
                dkh[h_lo:h_lo + n_suffix, h] += dkeys[:n_suffix]
                dvh[h_lo:h_lo + n_suffix, h] += dvals[:n_suffix]
                dks[b, h] += dkeys[n_suffix:n_suffix + nsk]
                dvs[b, h] += dvals[n_suffix:n_suffix + nsk]
    return dq, dkh, dvh, dks, dvs

