"""FLOP and byte accounting for Sketch Attention, STCA and the SequenceO1 cost model.

Counting convention (SequenceO1, App. G.1): a product of an m x r and an r x p
matrix costs 2mrp FLOPs; only GEMM-shaped work is counted, softmax and other
elementwise work is not.

The closed forms of App. G.2-G.7 are reproduced so that the printed per-target
numbers (43.076 and 0.67419 GFLOPs) and ratios (~49.94x, ~63.89x) can be
checked; the same convention gives the hot path's algorithmic FLOPs:
4 k L d per head of SA (App. G.3, affinity plus aggregation) and
4 T (L + k_s) d per head of STCA.
"""
from __future__ import annotations


def gemm(m: float, r: float, p: float) -> float:
    """App. G.1: FLOPs(UV) = 2 m r p for U in R^{m x r}, V in R^{r x p}."""
    return 2.0 * m * r * p


def swiglu(L: float, D: float, D_ff: float) -> float:
    """App. G.1: FFN(U) = (swish(U W_1) * (U W_g)) W_2 on L tokens, width D -> D_ff -> D."""
    return gemm(L, D, D_ff) + gemm(L, D, D_ff) + gemm(L, D_ff, D)


def stca_layer(L: float, D: float, h: float) -> float:
    """App. G.2: one STCA layer with single-query reordering, plus the history pre-FFN."""
    d_h = D / h
    attn = h * (gemm(1, D, d_h) + gemm(1, d_h, D) + gemm(1, D, L) + gemm(1, L, D)
                + gemm(1, D, d_h))
    return swiglu(L, D, 2 * D) + attn + gemm(1, D, D) + swiglu(1, D, 2 * D)


def stca(L: float, n_layers: float, D: float, h: float) -> float:
    """App. G.2: N_stca (12 L D^2 + 4 L D h + 20 D^2)."""
    return n_layers * stca_layer(L, D, h)


def sa_layer(L: float, L_s: float, d: float) -> float:
    """App. G.3: key projection, prototype projection, affinity, aggregation, sketch FFN."""
    return (gemm(L, d, d) + gemm(L_s, d, d) + gemm(L_s, d, L) + gemm(L_s, L, d)
            + swiglu(L_s, d, 2 * d))


def sa(L: float, n_layers: float, L_s: float, d: float) -> float:
    """App. G.3: N_sa (2 L d^2 + 14 L_s d^2 + 4 L_s L d)."""
    return n_layers * sa_layer(L, L_s, d)


def adapt(L_s: float, d: float, D: float) -> float:
    """App. G.4: the sketch adapter X^ = X~ W_A."""
    return gemm(L_s, d, D)


def flops_hit(L_s, d, D, h, n_stca) -> float:
    """App. G.4: a cache hit runs the adapter and STCA over the L_s sketch tokens."""
    return adapt(L_s, d, D) + stca(L_s, n_stca, D, h)


def expected(L, p_hit, L_s, d, D, h, n_sa, n_stca) -> float:
    """App. G.4: E[FLOPs](L) = hit + (1 - p_hit) SA(L)."""
    return flops_hit(L_s, d, D, h, n_stca) + (1.0 - p_hit) * sa(L, n_sa, L_s, d)


def stca_mrlb(L, R, n_stca, D, h) -> float:
    """App. G.6: only the history pre-FFN of STCA is shared across the R targets."""
    shared = n_stca * swiglu(L, D, 2 * D)
    return shared / R + (stca(L, n_stca, D, h) - shared)


def seqo1_mrlb(L, R, p_hit, L_s, d, D, h, n_sa, n_stca) -> float:
    """App. G.6: E[FLOPs^MRLB](L; R, p_hit) per target."""
    shared = n_stca * swiglu(L_s, D, 2 * D)
    per_target = stca(L_s, n_stca, D, h) - shared
    return per_target + (adapt(L_s, d, D) + shared + (1.0 - p_hit) * sa(L, n_sa, L_s, d)) / R


# App. G.5 instantiation.
PAPER = dict(d=128, h=16, D=1024, n_sa=2, L_s=1024, n_stca=4)


def paper_numbers(L: float = 100_000) -> dict:
    """The App. G.7 comparison at L = 100K with the G.5 hyper-parameters."""
    p = PAPER
    stca_infer = stca_mrlb(L, 300, p["n_stca"], p["D"], p["h"])
    seqo1_infer = seqo1_mrlb(L, 300, 0.6, p["L_s"], p["d"], p["D"], p["h"], p["n_sa"], p["n_stca"])
    stca_train = stca_mrlb(L, 40, p["n_stca"], p["D"], p["h"])
    seqo1_train = seqo1_mrlb(L, 40, 0.5, p["L_s"], p["d"], p["D"], p["h"], p["n_sa"], p["n_stca"])
    stca_plain = stca(L, p["n_stca"], p["D"], p["h"])
    seqo1_plain = expected(L, 0.5, p["L_s"], p["d"], p["D"], p["h"], p["n_sa"], p["n_stca"])
    return {
        "stca_infer_gflops_per_target": stca_infer / 1e9,
        "seqo1_infer_gflops_per_target": seqo1_infer / 1e9,
        "ratio_infer": stca_infer / seqo1_infer,
        "ratio_train_mrlb": stca_train / seqo1_train,
        "ratio_no_mrlb": stca_plain / seqo1_plain,
        "sa_two_layers_gflops": sa(L, p["n_sa"], p["L_s"], p["d"]) / 1e9,
    }


# Hot-path accounting (algorithmic, per launch).

def sa_forward_flops(valid_tokens: int, heads: int, protos: int, head_dim: int) -> float:
    """Affinity plus aggregation GEMMs: 4 k L d per head (App. G.3 dominant term)."""
    return 4.0 * protos * head_dim * heads * valid_tokens


def sa_backward_flops(valid_tokens: int, heads: int, protos: int, head_dim: int,
                      recompute: bool = True) -> float:
    """Recompute S (2kLd), dV, dA, dK, dQ (8kLd): 10 k L d per head with the recompute."""
    return (10.0 if recompute else 8.0) * protos * head_dim * heads * valid_tokens


def sa_forward_bytes(valid_tokens: int, heads: int, protos: int, head_dim: int, users: int,
                     in_bytes: int = 2, norm: int = 0, q_users: int = 1, kv_alias: bool = False) -> float:
    """K and V read once (one tensor when the values are the keys, the paper's V = X), Q read once,
    sketch written once (fp32), plus the saved lse."""
    kv = (1.0 if kv_alias else 2.0) * valid_tokens * heads * head_dim * in_bytes
    q = float(q_users) * heads * protos * head_dim * in_bytes
    out = 4.0 * users * heads * protos * head_dim
    lse = 4.0 * valid_tokens * heads if norm == 0 else 4.0 * users * heads * protos
    return kv + q + out + lse


def stca_forward_flops(total_targets: int, keys_per_target: float, heads: int,
                       head_dim: int) -> float:
    return 4.0 * total_targets * keys_per_target * heads * head_dim


def refine_flops(rows: float, d: float, project: bool = True) -> float:
    """One refinement of `rows` sketch rows (all users and heads) of width d (§3.3, Eq. (13)-(14)):
    the SwiGLU FFN at width 2d (App. G.3's 12 L_s d^2) and, with `project`, the next layer's query
    projection X~ W_Q (App. G.3's 2 L_s d^2)."""
    return swiglu(rows, d, 2 * d) + (gemm(rows, d, d) if project else 0.0)


def refine_bytes(rows: float, heads: float, d: float, project: bool = True) -> float:
    """Bytes a refinement moves at least once: x_tilde and x_hat read and x_next written in fp32,
    q_next written in bf16, and the weights (bf16) and LayerNorm vectors (fp32) of every head."""
    weights = heads * (3 * d * 2 * d + (d * d if project else 0)) * 2 + heads * 4 * d * 4
    return rows * d * (4 + 4 + 4 + (2 if project else 0)) + weights

