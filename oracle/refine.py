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
"""
from __future__ import annotations

import numpy as np

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
