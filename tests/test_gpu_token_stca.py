"""GPU parity of the row-softmax engine against the fp64 oracle: token-wise SA (the §5.1 Table 1
comparator) and STCA (§2.3 / §3.4 / §4.2). Same tolerance as the PROTO tests: max abs error
<= 1e-2 and relative L2 error <= 5e-3 on every output."""
import math

import numpy as np
import pytest
import torch

import oracle
from sketch_attention_flashsa_b200 import workloads as W

from test_gpu_sa_forward import _full_parity, assert_close, f64, run_gpu, run_oracle

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


def test_token_mass_is_one_per_prototype():
    """Token-wise: each prototype's weights sum to 1 over its user's valid tokens (0 for an empty
    user), so mass is exactly that."""
    inp = W.make_sa([300, 0, 129, 50], 2, 64, 256, seed=33, seqused=[300, 0, 100, 0], norm=W.NORM_TOKEN)
    sk, lse, ms = run_gpu(inp, norm="token", mass=True)
    osk, olse, oms = run_oracle(inp, W.NORM_TOKEN)
    assert_close(sk, osk, "token sketch")
    assert_close(ms, oms, "token mass")
    assert (ms[[0, 2]] == 1.0).all() and (ms[[1, 3]] == 0.0).all()


@pytest.mark.parametrize("d,k", [(64, 256), (128, 512)])
def test_token_keys_alias_values(d, k):
    inp = W.make_sa([700, 129, 1], 2, d, k, seed=34 + d, norm=W.NORM_TOKEN)
    sk, lse = run_gpu(inp, norm="token", alias=True)
    osk, olse, _ = run_oracle(inp, W.NORM_TOKEN, alias=True)
    assert_close(sk, osk, "token sketch (k is v)")
    assert_close(lse, olse, "token lse (k is v)")


def test_token_large_values_match():
    """bf16 weights times bf16 values accumulate in fp32: |v| beyond the fp16 range is fine."""
    inp = W.make_sa([900, 300], 2, 128, 256, seed=35, norm=W.NORM_TOKEN)
    s = 3.0e4
    big = W.SAInputs(inp.q, inp.k, (inp.v.float() * s).bfloat16(), inp.cu_seqlens, None, inp.scale, inp.norm)
    sk, lse = run_gpu(big, norm="token")
    osk, olse, _ = run_oracle(big, W.NORM_TOKEN)
    assert_close(sk, osk, "token sketch (|v| > 65504)", scale=s)
    assert_close(lse, olse, "token lse")


@pytest.mark.slow
def test_token_config2_full():
    _full_parity(W.config2(W.NORM_TOKEN), W.NORM_TOKEN)


@pytest.mark.slow
def test_token_config3_full():
    _full_parity(W.config3(W.NORM_TOKEN), W.NORM_TOKEN)


@pytest.mark.slow
def test_token_config3_masked_full():
    _full_parity(W.config3(W.NORM_TOKEN, masked=True), W.NORM_TOKEN)


# ---------------------------------------------------------------------------------- STCA
def run_stca(inp: W.STCAInputs, alias=False, max_targets=None, status=False):
    """alias: one device tensor for k_hist and v_hist and one for k_sk and v_sk (keys = values)."""
    api = _api()
    dev = "cuda"
    ks = inp.k_sk.to(dev) if inp.k_sk.shape[2] > 0 else None
    vs = (ks if alias else inp.v_sk.to(dev)) if inp.v_sk.shape[2] > 0 else None
    kvl = inp.target_kv_len.to(dev) if inp.target_kv_len is not None else None
    kh = inp.k_hist.to(dev)
    vh = kh if alias else inp.v_hist.to(dev)
    cut = inp.cu_targets.to(dev)
    desc = api.stca_desc(inp.q, inp.k_hist, ks, cut, inp.cu_hist, scale=inp.scale,
                         max_targets=max_targets if max_targets is not None else int(inp.q.shape[0]))
    ws = torch.empty(max(api.stca_forward_workspace_size(desc), 256), dtype=torch.uint8, device=dev)
    out, lse = api.stca_forward(inp.q.to(dev), cut, kh, vh, inp.cu_hist.to(dev), ks, vs, scale=inp.scale,
                                target_kv_len=kvl, max_targets=max_targets, workspace=ws)
    torch.cuda.synchronize()
    res = (out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64))
    return res + (api.read_device_status(ws),) if status else res


def oracle_stca(inp: W.STCAInputs, alias=False):
    kvl = inp.target_kv_len.numpy() if inp.target_kv_len is not None else None
    vh, vs = (inp.k_hist, inp.k_sk) if alias else (inp.v_hist, inp.v_sk)
    return oracle.stca_forward(f64(inp.q), inp.cu_targets.numpy(), f64(inp.k_hist), f64(vh),
                               inp.cu_hist.numpy(), f64(inp.k_sk), f64(vs), inp.scale, kvl)


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


def test_stca_keys_alias_values():
    inp = W.make_stca([200, 64], [900, 300], 2, 64, 128, seed=42, with_kv_len=True)
    out, lse = run_stca(inp, alias=True)
    oout, olse = oracle_stca(inp, alias=True)
    assert_close(out, oout, "stca out (k is v)")
    assert_close(lse, olse, "stca lse (k is v)")


def test_stca_too_small_max_targets_gives_nan_and_status():
    """max_targets below a user's target count: the schedule records SKA_ERR_INVALID_VALUE and the
    combine writes NaN to every output instead of partial slots that were never written."""
    inp = W.make_stca([300, 40], [500, 200], 2, 64, 16, seed=43)
    out, lse, st = run_stca(inp, max_targets=100, status=True)
    assert st == 1  # SKA_ERR_INVALID_VALUE
    assert np.isnan(out).all() and np.isnan(lse).all()
    out, lse = run_stca(inp)  # the next call on the same context is correct
    oout, olse = oracle_stca(inp)
    assert_close(out, oout, "stca out after a refused call")


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
def test_stca_config5_full():
    """Config 5 in full: every target of every user against the oracle."""
    inp = W.config5()
    out, lse = run_stca(inp)
    cut = inp.cu_targets.numpy()
    cuh = inp.cu_hist.numpy()
    for b in range(len(cut) - 1):
        rows = slice(int(cut[b]), int(cut[b + 1]))
        sub = W.STCAInputs(inp.q[rows], torch.tensor([0, cut[b + 1] - cut[b]], dtype=torch.int32),
                           inp.k_hist[cuh[b]:cuh[b + 1]], inp.v_hist[cuh[b]:cuh[b + 1]],
                           torch.tensor([0, cuh[b + 1] - cuh[b]], dtype=torch.int32), inp.k_sk[b:b + 1],
                           inp.v_sk[b:b + 1], inp.scale)
        oout, olse = oracle_stca(sub)
        assert_close(out[rows], oout, f"stca out user {b}")
        assert_close(lse[rows], olse, f"stca lse user {b}")
