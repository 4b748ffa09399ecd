"""GPU parity of the row-softmax engine against the fp64 oracle: token-wise SA (the §5.1 Table 1
comparator) and STCA (§2.3 / §3.4 / §4.2). Same tolerance as the PROTO tests: max abs error
<= 1e-2 and relative L2 error <= 5e-3 on every output."""
import math

import numpy as np
import pytest
import torch

import oracle
from sketch_attention_flashsa_b200 import workloads as W

from test_gpu_sa_forward import assert_close, f64, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


def _api():
    from sketch_attention_flashsa_b200 import api
    return api


def check_token(inp):
    sk, lse = run_gpu(inp, norm="token")
    osk, olse, _ = run_oracle(inp, W.NORM_TOKEN)
    assert_close(sk, osk, "token sketch")
    assert_close(lse, olse, "token lse")
    return sk, lse


TOKEN_CASES = {
    "d64_k256_ragged": ([1, 127, 128, 129, 700], 2, 64, 256),
    "d128_k512": ([300, 1, 513], 2, 128, 512),
    "d64_k16": ([1000, 5], 1, 64, 16),
    "d128_k192": ([640, 33], 3, 128, 192),
    "d64_k1024": ([257], 1, 64, 1024),
    # three query tiles: the second CTA of a group holds one query tile (second warpgroup idle)
    "d128_k384": ([520, 1, 129], 2, 128, 384),
}


@pytest.mark.parametrize("name", sorted(TOKEN_CASES))
def test_token_parity_small(name):
    lengths, H, d, k = TOKEN_CASES[name]
    check_token(W.make_sa(lengths, H, d, k, seed=300 + len(name), norm=W.NORM_TOKEN))


def test_token_config1_fp32():
    inp = W.config1()
    inp.norm = W.NORM_TOKEN
    check_token(inp)


def test_token_empty_padded_per_user_scale():
    inp = W.make_sa([200, 0, 300, 130], 2, 128, 256, seed=31, seqused=[150, 0, 1, 200], norm=W.NORM_TOKEN,
                    per_user_q=True, q_sigma=1.0, scale=1.0 / math.sqrt(128))
    sk, lse = check_token(inp)
    assert (sk[1] == 0).all() and np.isneginf(lse[1]).all()


def test_token_padding_bitwise_and_deterministic():
    inp = W.make_sa([400, 300], 2, 64, 256, seed=32, seqused=[250, 300], norm=W.NORM_TOKEN)
    a, la = run_gpu(inp, norm="token")
    k2, v2 = inp.k.clone(), inp.v.clone()
    k2[250:400] = (torch.randn(150, 2, 64) * 50).bfloat16()
    v2[250:400] = (torch.randn(150, 2, 64) * 50).bfloat16()
    b, lb = run_gpu(W.SAInputs(inp.q, k2, v2, inp.cu_seqlens, inp.seqused, inp.scale, inp.norm), norm="token")
    assert np.array_equal(a, b) and np.array_equal(la, lb)
    c, lc = run_gpu(inp, norm="token")
    assert np.array_equal(a, c) and np.array_equal(la, lc)


@pytest.mark.slow
def test_token_config2_full_sampled():
    inp = W.config2(W.NORM_TOKEN)
    sk, lse = run_gpu(inp, norm="token")
    cu = inp.cu_seqlens.numpy()
    lens = inp.valid_lengths()
    q = f64(inp.q)
    for b, h in [(0, 0), (int(np.argmax(lens)), 3), (63, 1)]:
        lo, n = int(cu[b]), int(lens[b])
        osk, olse, _, _ = oracle.sa_problem(q[h], f64(inp.k[lo:lo + n, h]), f64(inp.v[lo:lo + n, h]), inp.scale,
                                            W.NORM_TOKEN)
        assert_close(sk[b, h], osk, f"token sketch[{b},{h}]")
        assert_close(lse[b, h], olse, f"token lse[{b},{h}]")


@pytest.mark.slow
def test_token_config3_full_sampled():
    inp = W.config3(W.NORM_TOKEN)
    sk, lse = run_gpu(inp, norm="token")
    q = f64(inp.q)
    for b, h in [(0, 0), (7, 5)]:
        lo = b * 100_000
        osk, olse, _, _ = oracle.sa_problem(q[h], f64(inp.k[lo:lo + 100_000, h]), f64(inp.v[lo:lo + 100_000, h]),
                                            inp.scale, W.NORM_TOKEN)
        assert_close(sk[b, h], osk, f"token sketch[{b},{h}]")
        assert_close(lse[b, h], olse, f"token lse[{b},{h}]")


# ---------------------------------------------------------------------------------- STCA
def run_stca(inp: W.STCAInputs):
    api = _api()
    dev = "cuda"
    ks = inp.k_sk.to(dev) if inp.k_sk.shape[2] > 0 else None
    vs = inp.v_sk.to(dev) if inp.v_sk.shape[2] > 0 else None
    kvl = inp.target_kv_len.to(dev) if inp.target_kv_len is not None else None
    out, lse = api.stca_forward(inp.q.to(dev), inp.cu_targets.to(dev), inp.k_hist.to(dev), inp.v_hist.to(dev),
                                inp.cu_hist.to(dev), ks, vs, scale=inp.scale, target_kv_len=kvl)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def oracle_stca(inp: W.STCAInputs):
    kvl = inp.target_kv_len.numpy() if inp.target_kv_len is not None else None
    return oracle.stca_forward(f64(inp.q), inp.cu_targets.numpy(), f64(inp.k_hist), f64(inp.v_hist),
                               inp.cu_hist.numpy(), f64(inp.k_sk), f64(inp.v_sk), inp.scale, kvl)


STCA_CASES = {
    # (targets per user, suffix per user, sketch rows, heads, d, kv_len)
    "ragged_d64_ks256": ([1, 130, 256], [0, 300, 129], 256, 2, 64, False),
    "d128_ks16": ([200, 7], [1000, 64], 16, 2, 128, False),
    "no_sketch": ([129, 40], [500, 1], 0, 4, 64, False),
    "kv_len_mask": ([150, 60], [700, 300], 100, 2, 64, True),
    "only_sketch": ([64], [0], 256, 1, 128, False),
    # users with 3, 1 and 3 query tiles: pairs with and without a second query tile alternate
    # along one CTA's key columns
    "odd_tiles_mixed": ([300, 100, 257], [400, 900, 130], 64, 2, 128, True),
}


@pytest.mark.parametrize("name", sorted(STCA_CASES))
def test_stca_parity_small(name):
    tg, hist, ks, H, d, kvl = STCA_CASES[name]
    inp = W.make_stca(tg, hist, H, d, ks, seed=400 + len(name), with_kv_len=kvl)
    out, lse = run_stca(inp)
    oout, olse = oracle_stca(inp)
    assert_close(out, oout, "stca out")
    assert_close(lse, olse, "stca lse")


def test_stca_merge_law_on_gpu():
    """[suffix ; sketch] in one call equals the lse-weighted merge of the two one-segment calls."""
    inp = W.make_stca([300, 100], [2000, 700], 2, 64, 256, seed=41)
    out, lse = run_stca(inp)
    empty = torch.zeros((2, 2, 0, 64), dtype=torch.bfloat16)
    a = W.STCAInputs(inp.q, inp.cu_targets, inp.k_hist, inp.v_hist, inp.cu_hist, empty, empty, inp.scale)
    no_hist = torch.zeros((0, 2, 64), dtype=torch.bfloat16)
    b = W.STCAInputs(inp.q, inp.cu_targets, no_hist, no_hist, torch.zeros(3, dtype=torch.int32), inp.k_sk,
                     inp.v_sk, inp.scale)
    o1, l1 = run_stca(a)
    o2, l2 = run_stca(b)
    lm = np.logaddexp(l1, l2)
    merged = np.exp(l1 - lm)[..., None] * o1 + np.exp(l2 - lm)[..., None] * o2
    assert np.abs(merged - out).max() < 2e-3 and np.abs(lm - lse).max() < 1e-4


@pytest.mark.slow
def test_stca_config5_full_sampled():
    inp = W.config5()
    out, lse = run_stca(inp)
    cut = inp.cu_targets.numpy()
    cuh = inp.cu_hist.numpy()
    rng = np.random.default_rng(5)
    for b in (0, 7, 15):
        rows = np.sort(rng.choice(np.arange(cut[b], cut[b + 1]), size=12, replace=False))
        sub = W.STCAInputs(inp.q[rows], torch.tensor([0, len(rows)], dtype=torch.int32),
                           inp.k_hist[cuh[b]:cuh[b + 1]], inp.v_hist[cuh[b]:cuh[b + 1]],
                           torch.tensor([0, cuh[b + 1] - cuh[b]], dtype=torch.int32), inp.k_sk[b:b + 1],
                           inp.v_sk[b:b + 1], inp.scale)
        oout, olse = oracle_stca(sub)
        assert_close(out[rows], oout, f"stca out user {b}")
        assert_close(lse[rows], olse, f"stca lse user {b}")
