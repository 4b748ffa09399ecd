"""fp64 oracle for the stacked refinement of the sketch (SequenceO1 §3.3).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: SequenceO1 (arXiv 2609.08443), §3.3 "Stacked Refinement", Eq. (10)-(14): layer l takes
the sketch X~(l), recomputes the affinities with per-user queries X~(l) W_Q(l) (Eq. (10)-(11),
the SA forward with per-user prototypes), aggregates X^(l+1) = A(l) X (Eq. (12)) and refines
  Eq. (13)  X-(l+1) = LN(X~(l) + X^(l+1))
  Eq. (14)  X~(l+1) = LN(X-(l+1) + FFN(X-(l+1)))
with the SwiGLU FFN of App. G.1 (FFN(U) = (swish(U W_1) * (U W_g)) W_2) at intermediate width 2d
(App. G.3, "Sketch FFN").

Readings taken here (the pages name LN and the FFN but not their details):
* LN normalises each sketch token (row) over its d features: (x - mean) / sqrt(var + eps) with
  the biased variance and eps = 1e-5, then the affine gamma * . + beta (gamma = 1, beta = 0 when
  not given).
* swish(u) = u * sigmoid(u) (swish with beta = 1, i.e. SiLU).
* H heads are H independent problems on d-wide slices, each with its own LN and FFN parameters
  (the paper's SA is single-head: H = 1).
* X~^(0) = P^(0): layer 0's input sketch is the prototype matrix itself, the same for every user, so
  that S^(0) of Eq. (10) is Eq. (7)'s (P^(0) W_Q)(X W_K)^T and its residual in Eq. (13) adds P^(0).
* The keys K^(l) = X W_K^(l) of each layer are inputs (the key projection of the history is not
  part of this oracle); the values are X itself (Eq. (9), Eq. (12)).
* Optionally (``query_bf16``) each layer's queries X~^(l) W_Q^(l) are rounded to bf16 before the
  SA step, the input precision of SA (bf16 inputs, fp32 softmax); everything else stays fp64.
"""
from __future__ import annotations

import numpy as np

from .sa import NORM_PROTO, sa_forward

LN_EPS = 1e-5


def layer_norm(x, gamma=None, beta=None, eps=LN_EPS):
    """Row-wise LayerNorm over the last axis (float64)."""
    x = np.asarray(x, dtype=np.float64)
    mean = x.mean(axis=-1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=-1, keepdims=True)
    y = (x - mean) / np.sqrt(var + eps)
    if gamma is not None:
        y = y * np.asarray(gamma, dtype=np.float64)
    if beta is not None:
        y = y + np.asarray(beta, dtype=np.float64)
    return y


def swish(u):
    """swish(u) = u * sigmoid(u)."""
    u = np.asarray(u, dtype=np.float64)
    return u / (1.0 + np.exp(-u))


def swiglu_ffn(x, w1, wg, w2):
    """App. G.1: FFN(U) = (swish(U W_1) * (U W_g)) W_2; x [..., d], w1, wg [d, f], w2 [f, d]."""
    x = np.asarray(x, dtype=np.float64)
    return (swish(x @ np.asarray(w1, np.float64)) * (x @ np.asarray(wg, np.float64))) @ np.asarray(w2, np.float64)


def refine(x_tilde, x_hat, w1, wg, w2, gamma1=None, beta1=None, gamma2=None, beta2=None):
    """Eq. (13)-(14) for a batch of sketches.

    x_tilde, x_hat: [B, H, k, d] (the previous sketch and this layer's aggregation A X);
    w1, wg: [H, d, f]; w2: [H, f, d]; gamma*, beta*: [H, d] or None.
    Returns (x_bar [B, H, k, d], x_tilde_next [B, H, k, d]).
    """
    x_tilde = np.asarray(x_tilde, dtype=np.float64)
    x_hat = np.asarray(x_hat, dtype=np.float64)
    B, H, k, d = x_tilde.shape
    x_bar = np.zeros((B, H, k, d))
    out = np.zeros((B, H, k, d))
    for h in range(H):
        g1 = None if gamma1 is None else np.asarray(gamma1)[h]
        b1 = None if beta1 is None else np.asarray(beta1)[h]
        g2 = None if gamma2 is None else np.asarray(gamma2)[h]
        b2 = None if beta2 is None else np.asarray(beta2)[h]
        xb = layer_norm(x_tilde[:, h] + x_hat[:, h], g1, b1)              # Eq. (13)
        y = swiglu_ffn(xb, np.asarray(w1)[h], np.asarray(wg)[h], np.asarray(w2)[h])
        x_bar[:, h] = xb
        out[:, h] = layer_norm(xb + y, g2, b2)                            # Eq. (14)
    return x_bar, out


def project_queries(x, w_q):
    """Queries of one layer, X~^(l) W_Q^(l) (Eq. (10); Eq. (7) for the prototypes P^(0)), per head.

    x: [H, k, d] or [B, H, k, d]; w_q: [H, d, d]. Returns x's shape.
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w_q, dtype=np.float64)
    out = np.zeros(x.shape)
    for h in range(w.shape[0]):
        out[..., h, :, :] = x[..., h, :, :] @ w[h]
    return out


def round_bf16(x):
    """x rounded to the nearest bfloat16 value (8 significant bits, ties to even), returned as
    float64; finite normal range only (|x| well inside [2^-126, 2^127]), zeros kept."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.round(m * 256.0) / 256.0, e)  # np.round: half to even


def stacked_sa(p0, w_q, keys, v, cu_seqlens, seqused, scale, ffn, query_bf16=False):
    """N_sa stacked SA layers (§3.3, Eq. (10)-(14)), N_sa = len(w_q).

    p0: [H, k, d] prototypes P^(0) (= X~^(0), shared by all users); w_q: N_sa arrays [H, d, d];
    keys: N_sa arrays [T, H, d], K^(l) = X W_K^(l); v: [T, H, d] the history X (the values);
    ffn: N_sa tuples (w1, wg, w2, gamma1, beta1, gamma2, beta2) as in `refine`.
    Layer l: Q = X~^(l) W_Q^(l); X^^(l+1) = A^(l) X with A^(l) the prototype-wise softmax of
    scale Q K^(l)T (Eq. (10)-(12)); X~^(l+1) from Eq. (13)-(14).
    query_bf16: round each layer's queries to bf16 before its SA step (the SA input precision).
    Returns X~^(N_sa) as [B, H, k, d] and the per-layer sketches X^^(l+1).
    """
    p0 = np.asarray(p0, dtype=np.float64)
    B = len(cu_seqlens) - 1
    x_t = np.broadcast_to(p0, (B,) + p0.shape).copy()
    sketches = []
    for l in range(len(w_q)):
        q = project_queries(x_t, w_q[l])
        if query_bf16:
            q = round_bf16(q)
        x_hat, _, _ = sa_forward(q, keys[l], v, cu_seqlens, seqused, scale, NORM_PROTO)
        sketches.append(x_hat)
        _, x_t = refine(x_t, x_hat, *ffn[l])
    return x_t, sketches

