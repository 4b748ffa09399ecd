"""fp64 oracle for the Sketch Attention (SA) forward and backward.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: SequenceO1 (arXiv 2609.08443), §3.1 "Sketch Attention (SA)":
  Eq. (7)  S = (P W_Q)(X W_K)^T / sqrt(d)          in R^{k x n}
  Eq. (8)  A = softmax_proto(S), sum_{j=1..k} A_{j,i} = 1
  Eq. (9)  X~ = A X                                 in R^{k x d}
and §3.3 (the same normalisation in every refinement layer), §4.4 FlashSA
(fused; reaches the same X~ without storing S), App. A.4 (SA is fully
differentiable).

Readings of the pages taken here (each is also pinned by a test):
* q = P W_Q and k = X W_K are inputs (the projections are plain GEMMs outside
  the fused step); v is the value matrix, X itself in the paper (Eq. (9)).
* ``scale`` replaces 1/sqrt(d) so that callers can fold it into q.
* H heads are H independent single-head SA problems on d-wide slices.
* PROTO (the paper's Eq. (8)): softmax over the k prototypes for each valid
  history token i. TOKEN (the "vanilla attention" comparator of §5.1 Table 1):
  softmax over the valid history tokens for each prototype j.
* No renormalisation after the aggregation: X~ = A X exactly (Eq. (9)).
* Tokens past a user's valid length take no part: PROTO gives them a zero
  column of A; TOKEN excludes them from the softmax domain. An empty user gives
  a zero sketch, and in TOKEN mode lse = -inf.
"""
from __future__ import annotations

import numpy as np

NORM_PROTO = 0
NORM_TOKEN = 1


def _segments(cu_seqlens, seqused):
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    B = cu.shape[0] - 1
    out = []
    for b in range(B):
        lo, hi = int(cu[b]), int(cu[b + 1])
        n = hi - lo
        if seqused is not None:
            n = min(n, int(np.asarray(seqused)[b]))
        out.append((lo, max(n, 0)))
    return out


def _q_for(q, b, h):
    return q[h] if q.ndim == 3 else q[b, h]


def sa_problem(q_bh, k_bh, v_bh, scale, norm):
    """One (user, head) SA forward: returns (sketch [k,d], lse, mass [k], A [k,n]).

    q_bh [k,d], k_bh [n,d], v_bh [n,d], float64.
    PROTO: Eq. (7)-(9); lse has shape [n] (one per token, over prototypes).
    TOKEN: softmax over tokens per prototype; lse has shape [k].
    """
    kp = q_bh.shape[0]
    n = k_bh.shape[0]
    d = v_bh.shape[1]
    if n == 0:
        sketch = np.zeros((kp, d))
        mass = np.zeros(kp)
        if norm == NORM_PROTO:
            return sketch, np.zeros(0), mass, np.zeros((kp, 0))
        return sketch, np.full(kp, -np.inf), mass, np.zeros((kp, 0))
    # Eq. (7): affinities between every prototype j and every token i.
    S = scale * (q_bh @ k_bh.T)                      # [k, n]
    if norm == NORM_PROTO:
        # Eq. (8): prototype-wise softmax, normalised down each column (token).
        m = S.max(axis=0)                            # [n]
        lse = m + np.log(np.exp(S - m[None, :]).sum(axis=0))
        A = np.exp(S - lse[None, :])
    elif norm == NORM_TOKEN:
        # Comparator: token-wise softmax along each row (prototype).
        m = S.max(axis=1)                            # [k]
        lse = m + np.log(np.exp(S - m[:, None]).sum(axis=1))
        A = np.exp(S - lse[:, None])
    else:
        raise ValueError(norm)
    # Eq. (9): sketch construction, no renormalisation.
    sketch = A @ v_bh
    mass = A.sum(axis=1)
    return sketch, lse, mass, A


def sa_forward(q, k, v, cu_seqlens, seqused=None, scale=1.0, norm=NORM_PROTO):
    """Batched SA forward over ragged users.

    q: [H,k,d] (prototypes shared by all users) or [B,H,k,d]; k, v: [T,H,d].
    Returns sketch [B,H,k,d], lse (PROTO: [T,H] with -inf on padding rows;
    TOKEN: [B,H,k]) and mass [B,H,k] = sum_i A_{j,i}.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    segs = _segments(cu_seqlens, seqused)
    B, T, H, d = len(segs), k.shape[0], k.shape[1], k.shape[2]
    kp = q.shape[-2]
    sketch = np.zeros((B, H, kp, d))
    mass = np.zeros((B, H, kp))
    if norm == NORM_PROTO:
        lse = np.full((T, H), -np.inf)
    else:
        lse = np.full((B, H, kp), -np.inf)
    for b, (lo, n) in enumerate(segs):
        for h in range(H):
            sk, ls, ms, _ = sa_problem(_q_for(q, b, h), k[lo:lo + n, h], v[lo:lo + n, h],
                                       scale, norm)
            sketch[b, h] = sk
            mass[b, h] = ms
            if norm == NORM_PROTO:
                lse[lo:lo + n, h] = ls
            else:
                lse[b, h] = ls
    return sketch, lse, mass


def sa_forward_proto(q, k, v, cu_seqlens, seqused=None, scale=1.0):
    """SA forward with the paper's prototype-wise normalisation (§3.1 Eq. (8))."""
    return sa_forward(q, k, v, cu_seqlens, seqused, scale, NORM_PROTO)


def sa_forward_token(q, k, v, cu_seqlens, seqused=None, scale=1.0):
    """SA forward with token-wise ("vanilla attention", §5.1 Table 1) normalisation."""
    return sa_forward(q, k, v, cu_seqlens, seqused, scale, NORM_TOKEN)


def _backward_problem(q_bh, k_bh, v_bh, do_bh, scale, norm):
    """Gradients of <dO, X~> for one (user, head), by the chain rule through Eq. (7)-(9).

    Returns (dq [k,d], dk [n,d], dv [n,d]).
    """
    kp, n = q_bh.shape[0], k_bh.shape[0]
    if n == 0:
        return np.zeros_like(q_bh), np.zeros_like(k_bh), np.zeros_like(v_bh)
    _, _, _, A = sa_problem(q_bh, k_bh, v_bh, scale, norm)
    # Eq. (9) X~ = A V: dV = A^T dO and dA = dO V^T.
    dv = A.T @ do_bh                                   # [n, d]
    dA = do_bh @ v_bh.T                                # [k, n]
    # Softmax Jacobian along the normalised axis.
    if norm == NORM_PROTO:
        # column-wise softmax (over prototypes j, per token i)
        delta = (A * dA).sum(axis=0)                   # [n]
        dS = A * (dA - delta[None, :])
    else:
        # row-wise softmax (over tokens i, per prototype j)
        Dj = (A * dA).sum(axis=1)                      # [k]
        dS = A * (dA - Dj[:, None])
    # Eq. (7) S = scale q k^T.
    dq = scale * (dS @ k_bh)                           # [k, d]
    dk = scale * (dS.T @ q_bh)                         # [n, d]
    return dq, dk, dv


def sa_backward(q, k, v, cu_seqlens, seqused, dsketch, scale=1.0, norm=NORM_PROTO):
    """Batched SA backward. dq has q's shape ([H,k,d] summed over users when the
    prototypes are shared, else [B,H,k,d]); dk, dv are [T,H,d] with zero rows on
    padding tokens."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(dsketch, dtype=np.float64)
    segs = _segments(cu_seqlens, seqused)
    H = k.shape[1]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b, (lo, n) in enumerate(segs):
        for h in range(H):
            gq, gk, gv = _backward_problem(_q_for(q, b, h), k[lo:lo + n, h], v[lo:lo + n, h],
                                           do[b, h], scale, norm)
            if q.ndim == 3:
                dq[h] += gq
            else:
                dq[b, h] += gq
            dk[lo:lo + n, h] = gk
            dv[lo:lo + n, h] = gv
    return dq, dk, dv


def sa_backward_proto(q, k, v, cu_seqlens, seqused, dsketch, scale=1.0):
    return sa_backward(q, k, v, cu_seqlens, seqused, dsketch, scale, NORM_PROTO)


def sa_backward_token(q, k, v, cu_seqlens, seqused, dsketch, scale=1.0):
    return sa_backward(q, k, v, cu_seqlens, seqused, dsketch, scale, NORM_TOKEN)
