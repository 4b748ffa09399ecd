"""Pins for the fp64 oracle: facts fixed by the pages and by the mathematics.

None of these tests re-types the oracle's formulas. Each one checks a closed
form, a conservation law, a special case, an invariance or finite differences,
chosen so that a dropped term, a wrong sign or index, a transposed operand or
the wrong softmax axis fails at least one of them.

Source: SequenceO1 (arXiv 2609.08443) §3.1 Eq. (7)-(9) (SA), §2.3 (STCA),
§5.1 Table 1 (token-wise "vanilla" normalisation as the comparator).
"""
import math
from fractions import Fraction

import numpy as np
import torch
import pytest

import oracle
from oracle.sa import NORM_PROTO, NORM_TOKEN

RNG = np.random.default_rng(1234)


def _rand_problem(lengths, H=2, d=8, kp=5, per_user_q=False, seed=0, sigma_q=0.7):
    rng = np.random.default_rng(seed)
    T = int(sum(lengths))
    B = len(lengths)
    q = rng.standard_normal((B, H, kp, d) if per_user_q else (H, kp, d)) * sigma_q
    k = rng.standard_normal((T, H, d))
    v = rng.standard_normal((T, H, d))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    return q, k, v, cu


# ---------------------------------------------------------------- hand example
# d = 2. Keys are one-hot so that S_{j,i} = q_j[c(i)]: k_0 = e_0, k_1 = e_1,
# k_2 = e_0. Prototypes q_0 = (0, ln 2), q_1 = (ln 3, 0). Scores (rows j, cols i):
#   S = [[0, ln2, 0], [ln3, 0, ln3]]
# PROTO (down each column): exp -> [[1,2,1],[3,1,3]] -> A = [[1/4,2/3,1/4],[3/4,1/3,3/4]]
# TOKEN (along each row):   A = [[1/4,1/2,1/4],[3/7,1/7,3/7]]
# Values v_0 = (4,0), v_1 = (0,3), v_2 = (8,4).
HAND_Q = np.array([[[0.0, math.log(2.0)], [math.log(3.0), 0.0]]])      # [H=1,k=2,d=2]
HAND_K = np.array([[[1.0, 0.0]], [[0.0, 1.0]], [[1.0, 0.0]]])           # [T=3,H=1,d=2]
HAND_V = np.array([[[4.0, 0.0]], [[0.0, 3.0]], [[8.0, 4.0]]])
HAND_CU = np.array([0, 3])


def _frac(a):
    return np.array([[float(Fraction(x)) for x in row] for row in a])


def test_hand_example_proto():
    sk, lse, mass = oracle.sa_forward_proto(HAND_Q, HAND_K, HAND_V, HAND_CU)
    # sketch_0 = 1/4 v0 + 2/3 v1 + 1/4 v2 = (3, 3); sketch_1 = 3/4 v0 + 1/3 v1 + 3/4 v2 = (9, 4)
    np.testing.assert_allclose(sk[0, 0], [[3.0, 3.0], [9.0, 4.0]], rtol=0, atol=1e-12)
    np.testing.assert_allclose(mass[0, 0], [7 / 6, 11 / 6], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[:, 0], [math.log(4), math.log(3), math.log(4)], atol=1e-12)


def test_hand_example_token():
    sk, lse, mass = oracle.sa_forward_token(HAND_Q, HAND_K, HAND_V, HAND_CU)
    # sketch_0 = (1/4)(4,0) + (1/2)(0,3) + (1/4)(8,4) = (3, 5/2)
    # sketch_1 = (3/7)(4,0) + (1/7)(0,3) + (3/7)(8,4) = (36/7, 15/7)
    np.testing.assert_allclose(sk[0, 0], _frac([["3", "5/2"], ["36/7", "15/7"]]), atol=1e-12)
    np.testing.assert_allclose(mass[0, 0], [1.0, 1.0], atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], [math.log(4), math.log(7)], atol=1e-12)


def test_hand_example_backward_proto_value():
    # With dO = e_{j=0, c=0} the loss is sketch[0,0] = sum_i A_{0,i} v_i[0]; its
    # gradient w.r.t. v_i[0] is A_{0,i} = (1/4, 2/3, 1/4) and 0 for v_i[1].
    dO = np.zeros((1, 1, 2, 2))
    dO[0, 0, 0, 0] = 1.0
    _, _, dv = oracle.sa_backward_proto(HAND_Q, HAND_K, HAND_V, HAND_CU, None, dO)
    np.testing.assert_allclose(dv[:, 0, 0], [0.25, 2 / 3, 0.25], atol=1e-12)
    np.testing.assert_allclose(dv[:, 0, 1], 0.0, atol=1e-12)


# ---------------------------------------------------------- conservation laws
@pytest.mark.parametrize("scale", [1.0, 0.35])
def test_proto_conservation_identity_values(scale):
    """Eq. (8): with V = I the sketch is A itself, so each token's column sums to 1."""
    n, d, kp = 6, 8, 5
    q, k, _, cu = _rand_problem([n], H=1, d=d, kp=kp, seed=3)
    v = np.zeros((n, 1, d))
    for i in range(n):
        v[i, 0, i] = 1.0
    sk, _, _ = oracle.sa_forward_proto(q, k, v, cu, scale=scale)
    A = sk[0, 0, :, :n]
    np.testing.assert_allclose(A.sum(axis=0), 1.0, atol=1e-13)
    assert (A > 0).all()


def test_token_conservation_identity_values():
    """Token-wise comparator: with V = I each prototype's row of A sums to 1."""
    n, d, kp = 6, 8, 5
    q, k, _, cu = _rand_problem([n], H=1, d=d, kp=kp, seed=4)
    v = np.zeros((n, 1, d))
    for i in range(n):
        v[i, 0, i] = 1.0
    sk, _, mass = oracle.sa_forward_token(q, k, v, cu)
    np.testing.assert_allclose(sk[0, 0, :, :n].sum(axis=1), 1.0, atol=1e-13)
    np.testing.assert_allclose(mass, 1.0, atol=1e-13)


def test_proto_sum_over_prototypes_is_value_sum():
    """Summing Eq. (9) over j and using Eq. (8): sum_j X~_j = sum_i x_i (valid i only)."""
    lengths = [7, 1, 12]
    used = [5, 1, 12]
    q, k, v, cu = _rand_problem(lengths, H=3, d=8, kp=6, seed=5)
    sk, _, mass = oracle.sa_forward_proto(q, k, v, cu, used)
    for b in range(3):
        lo = cu[b]
        np.testing.assert_allclose(sk[b].sum(axis=1), v[lo:lo + used[b]].sum(axis=0), atol=1e-12)
        np.testing.assert_allclose(mass[b].sum(axis=1), used[b], atol=1e-12)


def test_token_ones_column():
    """TOKEN: a value column of all ones gives a sketch column of ones."""
    q, k, v, cu = _rand_problem([9, 4], H=2, d=8, kp=3, seed=6)
    v[:, :, 2] = 1.0
    sk, _, _ = oracle.sa_forward_token(q, k, v, cu)
    np.testing.assert_allclose(sk[:, :, :, 2], 1.0, atol=1e-13)


# ------------------------------------------------------------- special cases
def test_proto_single_prototype_is_sum_pooling():
    """k = 1: each token gives all its mass to the one prototype; X~ = sum_i x_i."""
    q, k, v, cu = _rand_problem([10, 3], H=2, d=8, kp=1, seed=7)
    sk, lse, _ = oracle.sa_forward_proto(q, k, v, cu, scale=0.5)
    for b in range(2):
        np.testing.assert_allclose(sk[b, :, 0], v[cu[b]:cu[b + 1]].sum(axis=0), atol=1e-12)
    # lse_i = the single score 0.5 <q, k_i>
    np.testing.assert_allclose(lse[:, 0], 0.5 * (k[:, 0] * q[0, 0][None, :]).sum(axis=1), atol=1e-12)


def test_proto_zero_queries_split_evenly():
    q, k, v, cu = _rand_problem([10], H=1, d=8, kp=4, seed=8)
    q[:] = 0.0
    sk, lse, mass = oracle.sa_forward_proto(q, k, v, cu)
    np.testing.assert_allclose(sk[0, 0], np.tile(v[:, 0].sum(axis=0) / 4, (4, 1)), atol=1e-12)
    np.testing.assert_allclose(lse[:, 0], math.log(4), atol=1e-13)
    np.testing.assert_allclose(mass, 10 / 4, atol=1e-12)


def test_token_zero_queries_mean_pooling():
    q, k, v, cu = _rand_problem([10], H=1, d=8, kp=4, seed=9)
    q[:] = 0.0
    sk, lse, _ = oracle.sa_forward_token(q, k, v, cu)
    np.testing.assert_allclose(sk[0, 0], np.tile(v[:, 0].mean(axis=0), (4, 1)), atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], math.log(10), atol=1e-13)


def test_token_single_token():
    q, k, v, cu = _rand_problem([1], H=2, d=8, kp=4, seed=10)
    sk, lse, _ = oracle.sa_forward_token(q, k, v, cu, scale=0.3)
    for h in range(2):
        np.testing.assert_allclose(sk[0, h], np.tile(v[0, h], (4, 1)), atol=1e-13)
        np.testing.assert_allclose(lse[0, h], 0.3 * q[h] @ k[0, h], atol=1e-13)


def test_proto_hard_assignment_limit():
    """Large scale: Eq. (8) tends to a one-hot assignment of each token to its best prototype."""
    q, k, v, cu = _rand_problem([40], H=1, d=8, kp=5, seed=11)
    scale = 1.0e5
    sk, _, mass = oracle.sa_forward_proto(q, k, v, cu, scale=scale)
    s = k[:, 0] @ q[0].T           # [n, k], an independent recomputation of the ordering only
    best = s.argmax(axis=1)
    gap = np.sort(s, axis=1)[:, -1] - np.sort(s, axis=1)[:, -2]
    assert gap.min() * scale > 60   # every token's runner-up weight is < e^-60
    want = np.zeros((5, 8))
    for i, j in enumerate(best):
        want[j] += v[i, 0]
    np.testing.assert_allclose(sk[0, 0], want, atol=1e-10)
    np.testing.assert_allclose(mass[0, 0], np.bincount(best, minlength=5), atol=1e-10)


def test_token_hard_assignment_limit():
    """Large scale: each prototype copies the value of its best-scoring token."""
    q, k, v, cu = _rand_problem([40], H=1, d=8, kp=5, seed=12)
    scale = 1.0e5
    sk, _, _ = oracle.sa_forward_token(q, k, v, cu, scale=scale)
    s = q[0] @ k[:, 0].T           # [k, n]
    best = s.argmax(axis=1)
    srt = np.sort(s, axis=1)
    assert ((srt[:, -1] - srt[:, -2]) * scale).min() > 60
    np.testing.assert_allclose(sk[0, 0], v[best, 0], atol=1e-10)


def test_empty_user():
    q, k, v, cu = _rand_problem([5, 0, 3], H=2, d=8, kp=3, seed=13)
    sk, lse, mass = oracle.sa_forward_proto(q, k, v, cu)
    assert (sk[1] == 0).all() and (mass[1] == 0).all()
    skt, lset, masst = oracle.sa_forward_token(q, k, v, cu)
    assert (skt[1] == 0).all() and np.isneginf(lset[1]).all()


# ------------------------------------------------------------ invariances
@pytest.mark.parametrize("norm", [NORM_PROTO, NORM_TOKEN])
def test_permutation_invariance(norm):
    """Eq. (7)-(9) have no positional term: permuting a user's tokens keeps the sketch."""
    q, k, v, cu = _rand_problem([11, 6], H=2, d=8, kp=4, seed=14)
    perm = np.concatenate([RNG.permutation(11), 11 + RNG.permutation(6)])
    a = oracle.sa_forward(q, k, v, cu, None, 0.9, norm)
    b = oracle.sa_forward(q, k[perm], v[perm], cu, None, 0.9, norm)
    np.testing.assert_allclose(a[0], b[0], atol=1e-12)
    if norm == NORM_PROTO:
        np.testing.assert_allclose(a[1][perm], b[1], atol=1e-12)


@pytest.mark.parametrize("norm", [NORM_PROTO, NORM_TOKEN])
def test_padding_has_no_effect(norm):
    q, k, v, cu = _rand_problem([9, 7], H=2, d=8, kp=4, seed=15)
    used = [6, 7]
    a = oracle.sa_forward(q, k, v, cu, used, 1.0, norm)
    k2, v2 = k.copy(), v.copy()
    k2[6:9] = 1e3
    v2[6:9] = -7e2
    b = oracle.sa_forward(q, k2, v2, cu, used, 1.0, norm)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    # and equals the problem with the padding cut away
    c = oracle.sa_forward(q, np.concatenate([k[:6], k[9:]]), np.concatenate([v[:6], v[9:]]),
                          [0, 6, 13], None, 1.0, norm)
    np.testing.assert_allclose(a[0], c[0], atol=1e-13)
    if norm == NORM_PROTO:
        assert np.isneginf(a[1][6:9]).all()


def test_users_are_independent():
    q, k, v, cu = _rand_problem([8, 5, 6], H=2, d=8, kp=3, seed=16)
    a = oracle.sa_forward_proto(q, k, v, cu)
    k2 = k.copy()
    k2[8:13] += 1.0
    b = oracle.sa_forward_proto(q, k2, v, cu)
    np.testing.assert_array_equal(a[0][[0, 2]], b[0][[0, 2]])
    assert not np.allclose(a[0][1], b[0][1])


def test_heads_are_independent_problems():
    q, k, v, cu = _rand_problem([8], H=3, d=8, kp=3, seed=17)
    full = oracle.sa_forward_proto(q, k, v, cu)
    one = oracle.sa_forward_proto(q[1:2], k[:, 1:2], v[:, 1:2], cu)
    np.testing.assert_allclose(full[0][:, 1:2], one[0], atol=1e-14)


def test_scale_folds_into_queries():
    q, k, v, cu = _rand_problem([8, 3], H=2, d=8, kp=3, seed=18)
    a = oracle.sa_forward_token(q, k, v, cu, scale=0.125)
    b = oracle.sa_forward_token(q * 0.125, k, v, cu, scale=1.0)
    np.testing.assert_allclose(a[0], b[0], atol=1e-13)


def test_per_user_queries_match_shared_when_equal():
    q, k, v, cu = _rand_problem([8, 3], H=2, d=8, kp=3, seed=19)
    qb = np.stack([q, q])
    np.testing.assert_allclose(oracle.sa_forward_proto(q, k, v, cu)[0],
                               oracle.sa_forward_proto(qb, k, v, cu)[0], atol=0)


# --------------------------------------------------------- finite differences
def _fd_check(norm, per_user_q):
    lengths, used = [5, 4], [4, 4]
    q, k, v, cu = _rand_problem(lengths, H=2, d=4, kp=3, per_user_q=per_user_q, seed=20)
    rng = np.random.default_rng(21)
    dO = rng.standard_normal((2, 2, 3, 4))
    scale = 0.8
    dq, dk, dv = oracle.sa_backward(q, k, v, cu, used, dO, scale, norm)

    def loss(q_, k_, v_):
        return float((oracle.sa_forward(q_, k_, v_, cu, used, scale, norm)[0] * dO).sum())

    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = x.copy(); xp[idx] += eps
            xm = x.copy(); xm[idx] -= eps
            args = {"q": (q, k, v), "k": (q, k, v), "v": (q, k, v)}[name]
            ap = list(args); am = list(args)
            pos = "qkv".index(name)
            ap[pos] = xp; am[pos] = xm
            num[idx] = (loss(*ap) - loss(*am)) / (2 * eps)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8, err_msg=name)
    # padding rows get zero gradient
    assert (dk[4] == 0).all() and (dv[4] == 0).all()


@pytest.mark.parametrize("norm", [NORM_PROTO, NORM_TOKEN])
def test_backward_finite_differences_shared_q(norm):
    _fd_check(norm, per_user_q=False)


@pytest.mark.parametrize("norm", [NORM_PROTO, NORM_TOKEN])
def test_backward_finite_differences_per_user_q(norm):
    _fd_check(norm, per_user_q=True)


# ---------------------------------------------------------------------- STCA
def _stca_problem(targets, hist, ks, H=2, d=8, seed=30):
    rng = np.random.default_rng(seed)
    B = len(targets)
    q = rng.standard_normal((sum(targets), H, d))
    kh = rng.standard_normal((sum(hist), H, d))
    vh = rng.standard_normal((sum(hist), H, d))
    ksk = rng.standard_normal((B, H, ks, d))
    vsk = rng.standard_normal((B, H, ks, d))
    cut = np.concatenate([[0], np.cumsum(targets)])
    cuh = np.concatenate([[0], np.cumsum(hist)])
    return q, cut, kh, vh, cuh, ksk, vsk


def test_stca_single_key_returns_its_value():
    q, cut, kh, vh, cuh, ksk, vsk = _stca_problem([3], [1], 0)
    out, lse = oracle.stca_forward(q, cut, kh, vh, cuh, ksk, vsk, 0.5)
    np.testing.assert_allclose(out, np.broadcast_to(vh[0], out.shape), atol=1e-14)
    np.testing.assert_allclose(lse, 0.5 * (q * kh[0][None]).sum(axis=2), atol=1e-13)


def test_stca_zero_query_is_mean_of_all_keys():
    q, cut, kh, vh, cuh, ksk, vsk = _stca_problem([2, 3], [5, 4], 3)
    q[:] = 0
    out, lse = oracle.stca_forward(q, cut, kh, vh, cuh, ksk, vsk, 1.0)
    for b, (t0, t1, h0, h1) in enumerate([(0, 2, 0, 5), (2, 5, 5, 9)]):
        allv = np.concatenate([vh[h0:h1], vsk[b].transpose(1, 0, 2)], axis=0)
        np.testing.assert_allclose(out[t0:t1], np.broadcast_to(allv.mean(axis=0), out[t0:t1].shape), atol=1e-13)
        np.testing.assert_allclose(lse[t0:t1], math.log(allv.shape[0]), atol=1e-13)


def test_stca_segment_merge_law():
    """Softmax over [suffix; sketch] = lse-weighted merge of the two one-segment results."""
    q, cut, kh, vh, cuh, ksk, vsk = _stca_problem([4, 2], [6, 3], 5)
    out, lse = oracle.stca_forward(q, cut, kh, vh, cuh, ksk, vsk, 0.7)
    o1, l1 = oracle.stca_forward(q, cut, kh, vh, cuh, ksk[:, :, :0], vsk[:, :, :0], 0.7)
    o2, l2 = oracle.stca_forward(q, cut, kh[:0], vh[:0], np.zeros_like(cuh), ksk, vsk, 0.7)
    lm = np.logaddexp(l1, l2)
    np.testing.assert_allclose(lse, lm, atol=1e-12)
    merged = np.exp(l1 - lm)[..., None] * o1 + np.exp(l2 - lm)[..., None] * o2
    np.testing.assert_allclose(out, merged, atol=1e-12)


def test_stca_equals_token_sa_with_one_prototype():
    """One target over one user's suffix is token-wise SA with that target as the only prototype."""
    q, cut, kh, vh, cuh, ksk, vsk = _stca_problem([1], [7], 0, H=2)
    out, lse = oracle.stca_forward(q, cut, kh, vh, cuh, ksk, vsk, 0.6)
    sk, lse_t, _ = oracle.sa_forward_token(q[0][:, None, :], kh, vh, cuh, None, 0.6)
    np.testing.assert_allclose(out[0], sk[0, :, 0], atol=1e-13)
    np.testing.assert_allclose(lse[0], lse_t[0, :, 0], atol=1e-13)


def test_stca_kv_len_is_truncation():
    q, cut, kh, vh, cuh, ksk, vsk = _stca_problem([1, 1], [6, 5], 2)
    out, lse = oracle.stca_forward(q, cut, kh, vh, cuh, ksk, vsk, 1.0, target_kv_len=[3, 5])
    o2, l2 = oracle.stca_forward(q, cut, np.concatenate([kh[:3], kh[6:]]),
                                 np.concatenate([vh[:3], vh[6:]]), [0, 3, 8], ksk, vsk, 1.0)
    np.testing.assert_allclose(out, o2, atol=1e-14)


def test_stca_no_keys():
    q, cut, kh, vh, cuh, ksk, vsk = _stca_problem([2], [0], 0)
    out, lse = oracle.stca_forward(q, cut, kh, vh, cuh, ksk, vsk, 1.0)
    assert (out == 0).all() and np.isneginf(lse).all()


# ---------------------------------------------------------------------------------- refinement
# SequenceO1 §3.3 Eq. (13)-(14) and the SwiGLU FFN of App. G.1: pins that a dropped term, a wrong
# axis or a transposed weight would break.

def test_layer_norm_rows_have_zero_mean_and_unit_variance():
    rng = np.random.default_rng(70)
    x = rng.normal(3.0, 5.0, size=(6, 128))
    y = oracle.layer_norm(x)
    assert np.abs(y.mean(axis=-1)).max() < 1e-12
    var = x.var(axis=-1)
    assert np.allclose(y.var(axis=-1), var / (var + 1e-5), rtol=1e-12)


def test_layer_norm_axis_affine_and_scale_invariance():
    rng = np.random.default_rng(71)
    x = rng.normal(size=(4, 16))
    g, b = rng.normal(size=16), rng.normal(size=16)
    base = oracle.layer_norm(x)
    assert np.allclose(oracle.layer_norm(x, g, b), base * g + b, atol=1e-14)
    # over the features of each row, not over the rows: rows are independent
    assert np.allclose(oracle.layer_norm(x[1:2]), base[1:2], atol=1e-14)
    # invariant to a positive scale and a shift of the row (up to the eps term, ~eps / var)
    assert np.allclose(oracle.layer_norm(7.0 * x + 3.0), base, atol=1e-4)
    # a constant row normalises to zero (then beta)
    assert np.allclose(oracle.layer_norm(np.full((1, 8), 2.5), None, np.arange(8.0)), np.arange(8.0))


def test_swish_closed_forms():
    assert oracle.swish(0.0) == 0.0
    assert abs(oracle.swish(1.0) - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15
    assert abs(oracle.swish(40.0) - 40.0) < 1e-12 and abs(oracle.swish(-40.0)) < 1e-15
    assert abs(oracle.swish(-1.0) + math.exp(-1.0) / (1.0 + math.exp(-1.0))) < 1e-15


def test_swiglu_ffn_hand_example():
    """d = 2, intermediate 2: x = [1, 2], W_1 = I, W_g = [[0, 1], [1, 0]], W_2 = I:
    x W_1 = [1, 2], x W_g = [2, 1], swish(x W_1) * x W_g = [2 swish(1), swish(2)].
    With W_1 and W_g swapped the activation falls on the other projection: [swish(2), 2 swish(1)]."""
    s1, s2 = 1.0 / (1.0 + math.exp(-1.0)), 2.0 / (1.0 + math.exp(-2.0))
    eye, swap = np.eye(2), np.array([[0.0, 1.0], [1.0, 0.0]])
    x = np.array([[1.0, 2.0]])
    assert np.allclose(oracle.swiglu_ffn(x, eye, swap, eye), [[2 * s1, s2]], atol=1e-15)
    assert np.allclose(oracle.swiglu_ffn(x, swap, eye, eye), [[s2, 2 * s1]], atol=1e-15)
    # the output projection: W_2 = [[1, 0], [1, 1]] sums the two gated features into the second output
    assert np.allclose(oracle.swiglu_ffn(x, eye, swap, np.array([[1.0, 0.0], [1.0, 1.0]])),
                       [[2 * s1 + s2, s2]], atol=1e-15)


def test_refine_with_zero_ffn_output_is_ln_of_the_residual_twice():
    """W_2 = 0 makes FFN = 0, so Eq. (14) is LN(LN(X~ + X^)): LayerNorm is idempotent up to eps."""
    rng = np.random.default_rng(72)
    B, H, k, d, f = 2, 2, 5, 16, 32
    xt, xh = rng.normal(size=(B, H, k, d)), rng.normal(size=(B, H, k, d))
    w1, wg = rng.normal(size=(H, d, f)), rng.normal(size=(H, d, f))
    w2 = np.zeros((H, f, d))
    xb, out = oracle.refine(xt, xh, w1, wg, w2)
    assert np.allclose(xb, oracle.layer_norm(xt + xh), atol=1e-14)
    assert np.allclose(out, xb, atol=1e-4)


def test_refine_heads_rows_and_users_are_independent():
    rng = np.random.default_rng(73)
    B, H, k, d, f = 3, 2, 4, 8, 16
    xt, xh = rng.normal(size=(B, H, k, d)), rng.normal(size=(B, H, k, d))
    w1, wg, w2 = rng.normal(size=(H, d, f)), rng.normal(size=(H, d, f)), rng.normal(size=(H, f, d)) / 4
    g1, b1, g2, b2 = (rng.normal(size=(H, d)) for _ in range(4))
    xb, out = oracle.refine(xt, xh, w1, wg, w2, g1, b1, g2, b2)
    # head 1 alone with its own parameters
    xb1, out1 = oracle.refine(xt[:, 1:], xh[:, 1:], w1[1:], wg[1:], w2[1:], g1[1:], b1[1:], g2[1:], b2[1:])
    assert np.allclose(out[:, 1:], out1, atol=1e-14)
    # a permutation of the sketch tokens permutes the output rows the same way
    perm = rng.permutation(k)
    _, outp = oracle.refine(xt[:, :, perm], xh[:, :, perm], w1, wg, w2, g1, b1, g2, b2)
    assert np.allclose(outp, out[:, :, perm], atol=1e-12)
    # the residual: x_bar is LN of the sum, so swapping the two inputs changes nothing
    xb_s, out_s = oracle.refine(xh, xt, w1, wg, w2, g1, b1, g2, b2)
    assert np.allclose(out_s, out, atol=1e-12)


# --------------------------------------------------------------------- stacked layers (§3.3)

def test_project_queries_hand_example():
    """Per head x W_Q^h, with x on the left: head 0 swaps the two features, head 1 is the upper
    triangular [[1, 2], [0, 1]] (its transpose would give [3, 1] instead of [1, 3])."""
    w = np.array([[[0.0, 1.0], [1.0, 0.0]], [[1.0, 2.0], [0.0, 1.0]]])
    x = np.array([[[1.0, 2.0]], [[1.0, 1.0]]])            # [H=2, k=1, d=2]
    q = oracle.project_queries(x, w)
    assert np.array_equal(q, [[[2.0, 1.0]], [[1.0, 3.0]]])
    # per-user rows [B, H, k, d] use the same weights for every user
    xb = np.stack([x, 2 * x])
    assert np.array_equal(oracle.project_queries(xb, w), np.stack([q, 2 * q]))


def _ln2(a, b, eps=1e-5):
    """LayerNorm of the 2-vector [a, b] (no affine): [-c, c] * sign(b - a), c = h / sqrt(h^2 + eps)."""
    h = (b - a) / 2.0
    c = h / math.sqrt(h * h + eps)
    return -c, c


def test_stacked_sa_one_prototype_hand_worked():
    """k = 1: every token gives all its weight to the single prototype, so each layer's sketch is
    the sum of the values, [1, 2] + [3, 4] = [4, 6], whatever the queries and keys. With W_2 = 0
    each layer is LN(LN(residual)); layer 0's LN2 has beta = [10, 0]. Layer 0: [1, 0] + [4, 6] ->
    two LNs -> [-c, c] + [10, 0]; layer 1 adds [4, 6] to that (not to P^(0)), which flips the sign
    of the normalised difference."""
    p0 = np.array([[[1.0, 0.0]]])                         # [H=1, k=1, d=2]
    v = np.array([[[1.0, 2.0]], [[3.0, 4.0]]])            # [T=2, H=1, d=2]
    rng = np.random.default_rng(80)
    keys = [rng.normal(size=(2, 1, 2)) for _ in range(2)]
    w_q = [rng.normal(size=(1, 2, 2)) for _ in range(2)]
    w1, wg, w2 = rng.normal(size=(1, 2, 4)), rng.normal(size=(1, 2, 4)), np.zeros((1, 4, 2))
    ffn0 = (w1, wg, w2, None, None, None, np.array([[10.0, 0.0]]))
    ffn1 = (w1, wg, w2, None, None, None, None)
    out, sketches = oracle.stacked_sa(p0, w_q, keys, v, np.array([0, 2]), None, 1.0, [ffn0, ffn1])
    for s in sketches:
        assert np.allclose(s, [[[[4.0, 6.0]]]], atol=1e-14)
    a, b = _ln2(1.0 + 4.0, 0.0 + 6.0)
    a, b = _ln2(a, b)
    x1 = (a + 10.0, b)
    a, b = _ln2(x1[0] + 4.0, x1[1] + 6.0)
    a, b = _ln2(a, b)
    assert np.allclose(out, [[[[a, b]]]], atol=1e-12)
    assert a > 0 > b


def test_stacked_sa_zero_queries_average_the_values():
    """W_Q = 0 in every layer: all scores are 0, every token splits its weight evenly over the k
    prototypes, and each layer's sketch row is (1 / k) sum_i x_i for every prototype."""
    rng = np.random.default_rng(81)
    H, k, d, f = 2, 3, 4, 8
    lens = [5, 2]
    cu = np.array([0, 5, 7])
    v = rng.normal(size=(7, H, d))
    keys = [rng.normal(size=(7, H, d)) for _ in range(2)]
    w_q = [np.zeros((H, d, d))] * 2
    ffn = [(rng.normal(size=(H, d, f)), rng.normal(size=(H, d, f)), rng.normal(size=(H, f, d)),
            None, None, None, None)] * 2
    _, sketches = oracle.stacked_sa(rng.normal(size=(H, k, d)), w_q, keys, v, cu, None, 1.0, ffn)
    for s in sketches:
        for b, (lo, n) in enumerate(zip(cu[:-1], lens)):
            want = v[lo:lo + n].sum(axis=0) / k                # [H, d]
            assert np.allclose(s[b], np.broadcast_to(want[:, None, :], (H, k, d)), atol=1e-13)


def test_stacked_sa_token_order_and_users():
    """The stack sees a user's history as a set (the same permutation of keys and values leaves
    every layer unchanged), and users do not interact."""
    rng = np.random.default_rng(82)
    H, k, d, f = 1, 4, 8, 16
    cu = np.array([0, 6, 9])
    v = rng.normal(size=(9, H, d))
    keys = [rng.normal(size=(9, H, d)) for _ in range(2)]
    w_q = [rng.normal(size=(H, d, d)) / 3 for _ in range(2)]
    ffn = [(rng.normal(size=(H, d, f)) / 3, rng.normal(size=(H, d, f)) / 3, rng.normal(size=(H, f, d)) / 3,
            1 + rng.normal(size=(H, d)) / 10, rng.normal(size=(H, d)) / 10,
            1 + rng.normal(size=(H, d)) / 10, rng.normal(size=(H, d)) / 10) for _ in range(2)]
    p0 = rng.normal(size=(H, k, d))
    out, _ = oracle.stacked_sa(p0, w_q, keys, v, cu, None, 0.5, ffn)
    perm = np.concatenate([rng.permutation(6), 6 + rng.permutation(3)])
    outp, _ = oracle.stacked_sa(p0, w_q, [kk[perm] for kk in keys], v[perm], cu, None, 0.5, ffn)
    assert np.allclose(outp, out, atol=1e-12)
    v2 = v.copy()
    v2[6:] += rng.normal(size=(3, H, d))  # (a shift equal on every feature would be absorbed by LN)
    out2, _ = oracle.stacked_sa(p0, w_q, keys, v2, cu, None, 0.5, ffn)
    assert np.array_equal(out2[0], out[0]) and not np.allclose(out2[1], out[1])


def test_round_bf16_hand_cases_ties_to_even():
    """bf16 keeps 8 significant bits: near 1 the spacing is 2^-7. 1 + 2^-8 is halfway between 1
    (even mantissa) and 1 + 2^-7, so it goes to 1; 1 + 3 2^-8 is halfway between 1 + 2^-7 (odd) and
    1 + 2^-6 (even), so it goes up; a hair above a tie rounds up; signs are symmetric."""
    x = np.array([1 + 2.0**-8, 1 + 3 * 2.0**-8, 1 + 2.0**-8 + 2.0**-40, -(1 + 2.0**-8), 0.0, 3.0, 2.0**-20 * 255])
    want = np.array([1.0, 1 + 2.0**-6, 1 + 2.0**-7, -1.0, 0.0, 3.0, 2.0**-20 * 255])
    assert np.array_equal(oracle.round_bf16(x), want)


def test_round_bf16_matches_a_library_conversion_on_fp32_values():
    """On values that fp32 holds exactly, a single rounding to bf16 is what torch's fp32 -> bf16
    conversion (round to nearest even) computes."""
    rng = np.random.default_rng(83)
    x = (rng.standard_normal(200_000) * np.exp(rng.uniform(-30, 30, 200_000))).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    assert np.array_equal(oracle.round_bf16(x.astype(np.float64)), want)


def test_stacked_sa_bf16_queries_no_op_when_queries_are_bf16():
    """One layer with W_Q = I and bf16-valued prototypes: the queries are already bf16, so the
    rounding option changes nothing; with W_Q scaled by 1 + 2^-12 it does change the result."""
    rng = np.random.default_rng(84)
    H, k, d, f = 2, 3, 8, 16
    cu = np.array([0, 5, 9])
    v = rng.normal(size=(9, H, d))
    keys = [rng.normal(size=(9, H, d))]
    p0 = oracle.round_bf16(rng.normal(size=(H, k, d)))
    ffn = [(rng.normal(size=(H, d, f)) / 3, rng.normal(size=(H, d, f)) / 3, rng.normal(size=(H, f, d)) / 3,
            None, None, None, None)]
    eye = [np.broadcast_to(np.eye(d), (H, d, d)).copy()]
    a, _ = oracle.stacked_sa(p0, eye, keys, v, cu, None, 1.0, ffn)
    b, _ = oracle.stacked_sa(p0, eye, keys, v, cu, None, 1.0, ffn, query_bf16=True)
    assert np.array_equal(a, b)
    off = [eye[0] * (1 + 2.0**-12)]
    c, _ = oracle.stacked_sa(p0, off, keys, v, cu, None, 1.0, ffn)
    e, _ = oracle.stacked_sa(p0, off, keys, v, cu, None, 1.0, ffn, query_bf16=True)
    assert np.array_equal(e, a) and not np.array_equal(c, a)


# ------------------------------------------------------------------- STCA backward (finite differences)

@pytest.mark.parametrize("with_kv_len", [False, True])
def test_stca_backward_matches_finite_differences(with_kv_len):
    """Every gradient of <dO, out> against central differences of the forward oracle alone
    (h = 1e-6): the query of each target, the suffix keys and values shared by a user's targets
    (summed over them) and the sketch keys and values."""
    q, cut, kh, vh, cuh, ksk, vsk = _stca_problem([2, 3], [4, 5], 3, H=2, d=4, seed=44)
    kvl = np.array([2, 1, 0, 4, 3]) if with_kv_len else None
    rng = np.random.default_rng(45)
    do = rng.standard_normal(q.shape)
    scale = 0.7
    grads = oracle.stca_backward(q, cut, kh, vh, cuh, ksk, vsk, scale, do, kvl)

    def f(args):
        out, _ = oracle.stca_forward(args[0], cut, args[1], args[2], cuh, args[3], args[4], scale, kvl)
        return float((out * do).sum())

    base = [q, kh, vh, ksk, vsk]
    h = 1e-6
    for which, g in enumerate(grads):
        flat = base[which].reshape(-1)
        for idx in range(flat.size):
            plus = [x.copy() for x in base]
            minus = [x.copy() for x in base]
            plus[which].reshape(-1)[idx] += h
            minus[which].reshape(-1)[idx] -= h
            fd = (f(plus) - f(minus)) / (2 * h)
            assert abs(fd - g.reshape(-1)[idx]) < 1e-7, (which, idx, fd, g.reshape(-1)[idx])
    if with_kv_len:
        # suffix rows that no target of their user reaches get no gradient: rows 2, 3 of user 0
        # (lengths 2, 1) and the last row of user 1 (lengths 0, 4, 3)
        for rows in (slice(2, 4), slice(8, 9)):
            assert not grads[1][rows].any() and not grads[2][rows].any()
        assert grads[1][0:2].any() and grads[2][4:8].any()


# ------------------------------------------------------------- allocation diagnostics (Fig. 3, §2.4)

def test_token_max_weight_hand_example():
    """The hand example's PROTO columns are [1/4, 3/4], [2/3, 1/3], [1/4, 3/4]: maxima 3/4, 2/3, 3/4."""
    mw = oracle.token_max_weight(HAND_Q, HAND_K, HAND_V, HAND_CU)
    np.testing.assert_allclose(mw[:, 0], [0.75, 2.0 / 3.0, 0.75], atol=1e-15)


def test_token_max_weight_bounds_and_even_split():
    """Each token's weights sum to 1 over k prototypes, so its maximum lies in [1/k, 1]; with zero
    queries it is exactly 1/k. Padding rows carry -1."""
    q, k, v, cu = _rand_problem([7, 5], H=2, kp=5, seed=90)
    mw = oracle.token_max_weight(q, k, v, cu, [7, 3], 1.0)
    valid = np.r_[np.ones(7, bool), np.ones(3, bool), np.zeros(2, bool)]
    assert (mw[valid] >= 1 / 5 - 1e-15).all() and (mw[valid] <= 1).all()
    assert (mw[~valid] == -1).all()
    np.testing.assert_allclose(oracle.token_max_weight(np.zeros_like(q), k, v, cu)[:, :], 0.2, atol=1e-15)


def test_weight_histogram_counts():
    vals = np.array([0.0, 0.1, 0.5, 0.999, 1.0, 0.25, -1.0, -1.0])
    assert list(oracle.weight_histogram(vals, 4)) == [2, 1, 1, 2]   # [0,.25): 0, .1; [.25,.5): .25; ...
    assert oracle.weight_histogram(vals, 4).sum() == 6                 # padding (-1) is skipped


def test_renormalized_sketch_is_a_weighted_mean():
    """Hand example: sketch row j = sum_i A_ji v_i and mass_j = sum_i A_ji, so the renormalised
    row is the A-weighted mean of the values; with all values equal it is that value."""
    sk, _, mass = oracle.sa_forward_proto(HAND_Q, HAND_K, HAND_V, HAND_CU)
    r = oracle.renormalized_sketch(sk, mass)
    A = np.array([[0.25, 2 / 3, 0.25], [0.75, 1 / 3, 0.75]])
    want = (A @ HAND_V[:, 0]) / A.sum(axis=1)[:, None]
    np.testing.assert_allclose(r[0, 0], want, atol=1e-14)
    same = np.broadcast_to(np.array([[[2.0, -1.0]]]), HAND_V.shape)
    sk2, _, m2 = oracle.sa_forward_proto(HAND_Q, HAND_K, same, HAND_CU)
    np.testing.assert_allclose(oracle.renormalized_sketch(sk2, m2)[0, 0], [[2.0, -1.0]] * 2, atol=1e-14)
    assert not oracle.renormalized_sketch(np.ones((1, 1, 2, 3)), np.array([[[0.0, 2.0]]]))[0, 0, 0].any()


# ------------------------------------------------------------------------ sketch cache (§4.1)

def test_splitmix64_published_vectors():
    """The first three outputs of SplitMix64 from seed 0 (the generator's reference test vectors)."""
    g = 0x9E3779B97F4A7C15
    assert oracle.splitmix64(0) == 0xE220A8397B1DCDAF
    assert oracle.splitmix64(g) == 0x6E789E6AA1B965F4
    assert oracle.splitmix64((2 * g) & ((1 << 64) - 1)) == 0x06C45D188009454F


def test_cache_hand_worked_sequence():
    """One set of two ways, ttl 10: A at t=0 and B at t=1 both hit; C at t=2 evicts the oldest (A);
    at t=12 B (stored at 1) has expired, so D at t=12 takes B's way, not C's; re-putting C keeps
    its way and refreshes its time."""
    c = oracle.SketchCache(1, 2, 3, 10)
    A, B, C, D = (1, 7, 0, 100), (2, 7, 0, 100), (3, 7, 0, 100), (4, 7, 0, 100)
    row = lambda x: np.full(3, float(x))  # noqa: E731
    assert c.put([A, B], [row(1), row(2)], 0) == [0, 1]
    hits, rows = c.get([A, B, C], 1)
    assert list(hits) == [True, True, False] and rows[1][0] == 2.0
    assert c.put([C], [row(3)], 2) == [0]                 # A (time 0) is the oldest
    assert list(c.get([A, C], 2)[0]) == [False, True]
    assert list(c.get([B], 12)[0]) == [False]             # 12 - 1 > 10
    assert list(c.get([C], 12)[0]) == [True]              # 12 - 2 <= 10
    assert c.put([D], [row(4)], 12) == [1]                # B's way: expired before the oldest rule
    assert c.put([C], [row(5)], 13) == [0]                # same key, same way, new data and time
    hits, rows = c.get([C, D], 22)                          # 22 - 12 = 10: D still live
    assert list(hits) == [True, True] and rows[0][0] == 5.0 and rows[1][0] == 4.0
    assert list(c.get([C, D], 23)[0]) == [True, False]     # 23 - 12 > 10
    # at 24 both ways have expired: the first (way 0) takes A; a duplicate in the same batch is the
    # same key, so it lands on the same way and the later data wins
    assert c.put([A, A], [row(6), row(7)], 24) == [0, 0]
    assert c.get([A], 24)[1][0][0] == 7.0


def test_cache_keys_differ_by_every_field():
    """Version, configuration and history timestamp are all part of the key (a new model version or
    a newer history must not hit an old sketch)."""
    c = oracle.SketchCache(4, 4, 2, 100)
    base = (5, 1, 2, 3)
    c.put([base], [np.ones(2)], 0)
    for other in [(6, 1, 2, 3), (5, 2, 2, 3), (5, 1, 3, 3), (5, 1, 2, 4)]:
        assert not c.get([other], 0)[0][0]
    assert c.get([base], 0)[0][0]
