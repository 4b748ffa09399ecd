"""GPU parity of the SA forward (libska.so through its C ABI) against the fp64 oracle.

Tolerance (from the spec contract for bf16 inputs with fp32 accumulation): max abs error
<= 1e-2 and relative L2 error <= 5e-3 on every output, at every size tested. Inputs are the
seeded generators of sketch_attention_flashsa_b200.workloads, identical bits on both sides.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from sketch_attention_flashsa_b200 import workloads as W

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
REL_L2 = 5e-3


def _api():
    from sketch_attention_flashsa_b200 import api
    return api


def f64(t):
    return t.float().numpy().astype(np.float64)


def run_gpu(inp: W.SAInputs, norm="proto", mass=False, alias=False, status=False):
    """The CUDA path through the C ABI. alias: pass one device tensor as both k and v (the
    paper's V = X); status: also return the call's device status word."""
    api = _api()
    dev = "cuda"
    su = inp.seqused.to(dev) if inp.seqused is not None else None
    k = inp.k.to(dev)
    v = k if alias else inp.v.to(dev)
    desc = api.sa_desc(inp.q, inp.k, inp.cu_seqlens, scale=inp.scale, norm=norm)
    ws = torch.empty(api.sa_forward_workspace_size(desc), dtype=torch.uint8, device=dev)
    sk, lse, ms = api.sa_forward(inp.q.to(dev), k, v, inp.cu_seqlens.to(dev), su, scale=inp.scale, norm=norm,
                                 want_mass=mass, workspace=ws)
    torch.cuda.synchronize()
    out = [sk.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)]
    if mass:
        out.append(ms.cpu().numpy().astype(np.float64))
    if status:
        out.append(api.read_device_status(ws))
    return tuple(out)


def run_oracle(inp: W.SAInputs, norm=W.NORM_PROTO, alias=False):
    su = inp.seqused.numpy() if inp.seqused is not None else None
    v = inp.k if alias else inp.v
    return oracle.sa_forward(f64(inp.q), f64(inp.k), f64(v), inp.cu_seqlens.numpy(), su, inp.scale, norm)


def assert_close(got, want, what, scale=1.0):
    """max |got - want| <= 1e-2 * scale and ||got - want|| <= 5e-3 ||want||; `scale` is the size
    of the inputs when a test scales them (outputs scale with the values)."""
    assert got.shape == want.shape, (what, got.shape, want.shape)
    fin = np.isfinite(want)
    assert (np.isfinite(got) == fin).all(), f"{what}: finiteness differs"
    if not fin.any():
        return
    err = np.abs(got[fin] - want[fin])
    mx = float(err.max())
    denom = float(np.linalg.norm(want[fin]))
    rel = float(np.linalg.norm(got[fin] - want[fin]) / denom) if denom > 0 else float(np.linalg.norm(got[fin]))
    print(f"[parity] {what}: max abs {mx:.3e}, rel L2 {rel:.3e}, max |want| {np.abs(want[fin]).max():.3e}")
    assert mx <= MAX_ABS * scale and rel <= REL_L2, f"{what}: max abs {mx:.3e}, rel L2 {rel:.3e}"
    return mx, rel


def check_proto(inp):
    sk, lse = run_gpu(inp)
    osk, olse, _ = run_oracle(inp)
    assert_close(sk, osk, "sketch")
    # padding rows carry -inf on both sides
    assert_close(lse, olse, "lse")


CASES = {
    # (lengths, H, d, k): several tiles, ragged tails, one-token and exact-tile users
    "d64_k256_ragged": ([1, 127, 128, 129, 700], 2, 64, 256),
    "d128_k512_cluster2": ([300, 1, 513], 2, 128, 512),
    "d128_k1024_cluster4": ([257, 90], 1, 128, 1024),
    "d64_k16": ([1000, 5], 1, 64, 16),
    "d128_k64": ([640, 33], 3, 128, 64),
    "d64_k192": ([400], 2, 64, 192),
    "d128_k384_cluster2": ([200, 333], 1, 128, 384),
    "d64_k32": ([129], 4, 64, 32),
    "d128_k128": ([1200, 7, 64], 2, 128, 128),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_proto_parity_small(name):
    lengths, H, d, k = CASES[name]
    inp = W.make_sa(lengths, H, d, k, seed=100 + len(name))
    check_proto(inp)


def test_config1_fp32_inputs():
    check_proto(W.config1())


def test_scale_inv_sqrt_d():
    inp = W.make_sa([500, 260], 2, 128, 512, seed=7, q_sigma=1.0, scale=1.0 / math.sqrt(128))
    check_proto(inp)


def test_per_user_queries():
    inp = W.make_sa([300, 129, 40], 2, 64, 256, seed=8, per_user_q=True)
    check_proto(inp)
    inp = W.make_sa([300, 129], 2, 128, 512, seed=9, per_user_q=True)
    check_proto(inp)


def test_empty_and_padded_users():
    inp = W.make_sa([200, 0, 300, 130], 2, 64, 256, seed=10, seqused=[150, 0, 1, 200])
    sk, lse = run_gpu(inp)
    osk, olse, _ = run_oracle(inp)
    assert_close(sk, osk, "sketch")
    assert_close(lse, olse, "lse")
    assert (sk[1] == 0).all()
    assert np.isneginf(lse[200 + 1:500]).all() and np.isneginf(lse[150:200]).all()


def test_padding_contents_do_not_matter_bitwise():
    inp = W.make_sa([400, 300], 2, 128, 512, seed=11, seqused=[250, 300])
    sk1, l1 = run_gpu(inp)
    k2, v2 = inp.k.clone(), inp.v.clone()
    k2[250:400] = (torch.randn(150, 2, 128) * 50).bfloat16()
    v2[250:400] = (torch.randn(150, 2, 128) * 50).bfloat16()
    inp2 = W.SAInputs(inp.q, k2, v2, inp.cu_seqlens, inp.seqused, inp.scale, inp.norm)
    sk2, l2 = run_gpu(inp2)
    assert np.array_equal(sk1, sk2) and np.array_equal(l1, l2)


def test_users_independent_bitwise():
    inp = W.make_sa([300, 500, 200], 1, 64, 256, seed=12)
    sk1, _ = run_gpu(inp)
    k2 = inp.k.clone()
    k2[300:800] = (torch.randn(500, 1, 64)).bfloat16()
    sk2, _ = run_gpu(W.SAInputs(inp.q, k2, inp.v, inp.cu_seqlens, None, inp.scale, inp.norm))
    # users 0 and 2 are untouched; their partial sums may be split differently across clusters
    # only if the tile schedule changed, which it does not (lengths are equal)
    assert np.array_equal(sk1[[0, 2]], sk2[[0, 2]])
    assert not np.array_equal(sk1[1], sk2[1])


def test_deterministic():
    inp = W.make_sa([3000, 1700], 4, 64, 256, seed=13)
    a, la = run_gpu(inp)
    b, lb = run_gpu(inp)
    assert np.array_equal(a, b) and np.array_equal(la, lb)


def test_permutation_invariance():
    inp = W.make_sa([777], 2, 128, 512, seed=14)
    perm = torch.randperm(777)
    sk1, l1 = run_gpu(inp)
    inp2 = W.SAInputs(inp.q, inp.k[perm].contiguous(), inp.v[perm].contiguous(), inp.cu_seqlens, None,
                      inp.scale, inp.norm)
    sk2, l2 = run_gpu(inp2)
    assert np.abs(sk1 - sk2).max() < 2e-3
    assert np.abs(l1[perm.numpy()] - l2).max() < 1e-4


def _conservation(inp, sk, mass=None):
    """sum_j sketch[b,h,j,:] = sum of the user's valid value rows and sum_j mass[b,h,j] = its valid
    length (Eq. (8) summed into Eq. (9): every token's weights over the prototypes sum to 1)."""
    lens = inp.valid_lengths()
    cu = inp.cu_seqlens.numpy()
    v = inp.v.float()
    for b in range(len(lens)):
        want = v[cu[b]:cu[b] + lens[b]].double().sum(0).numpy()  # [H, d]
        got = sk[b].sum(axis=1)
        scale = max(1.0, float(np.abs(want).max()))
        assert np.abs(got - want).max() <= 1e-3 * scale * math.sqrt(max(lens[b], 1) / 1000 + 1), b
        if mass is not None:
            # each token's weights reach the aggregation through fp16 once (relative error up to
            # 2^-11 per token, independent across tokens: the sum drifts like sqrt(n)), and the
            # tensor core's accumulation within a mass chain of 8 tiles rounds toward zero (a bias
            # measured at 1.2e-5 of n for chains of 16 tiles, so about 6e-6 for 8)
            n = max(lens[b], 1)
            tol = 3 * 2.0**-11 * math.sqrt(n) + 1e-5 * n + 1e-3
            assert np.abs(mass[b].sum(axis=-1) - lens[b]).max() <= tol, b


def _full_parity(inp, norm=W.NORM_PROTO, mass=False):
    """Every (user, head) of a full-size workload against the oracle, one problem at a time."""
    got = run_gpu(inp, norm="proto" if norm == W.NORM_PROTO else "token", mass=mass)
    sk, lse = got[0], got[1]
    if norm == W.NORM_PROTO:
        _conservation(inp, sk, got[2] if mass else None)
    cu = inp.cu_seqlens.numpy()
    lens = inp.valid_lengths()
    q = f64(inp.q)
    worst = 0.0
    for b in range(inp.num_users):
        lo, n = int(cu[b]), int(lens[b])
        kb, vb = f64(inp.k[lo:lo + n]), f64(inp.v[lo:lo + n])
        for h in range(inp.num_heads):
            qb = q[h] if q.ndim == 3 else q[b, h]
            osk, olse, omass, _ = oracle.sa_problem(qb, kb[:, h], vb[:, h], inp.scale, norm)
            mx, _ = assert_close(sk[b, h], osk, f"sketch[{b},{h}]")
            worst = max(worst, mx)
            if norm == W.NORM_PROTO:
                assert_close(lse[lo:lo + n, h], olse, f"lse[{b},{h}]")
            else:
                assert_close(lse[b, h], olse, f"lse[{b},{h}]")
            if mass:
                assert_close(got[2][b, h], omass, f"mass[{b},{h}]")
    print(f"[parity] all {inp.num_users * inp.num_heads} (user, head) pairs, worst sketch max abs {worst:.3e}")
    return got


@pytest.mark.slow
def test_config2_full():
    _full_parity(W.config2())


@pytest.mark.slow
def test_config3_full():
    _full_parity(W.config3())


@pytest.mark.slow
def test_config3_masked_full():
    got = _full_parity(W.config3(masked=True))
    assert np.isneginf(got[1][70_000:100_000]).all()


@pytest.mark.slow
def test_config3_mass_full():
    """The mass output at the headline size: Sum_j mass = 100,000 per (user, head), and every entry
    against the oracle's sum of weights (the long chains are where fp32 accumulation drifts)."""
    inp = W.make_sa([100_000] * 2, 2, 128, 512, seed=2)
    _full_parity(inp, mass=True)


MASS_CASES = {
    # (lengths, H, d, k, seqused)
    "d64_k256_ragged_padded": ([1, 127, 0, 129, 700], 2, 64, 256, [1, 100, 0, 129, 650]),
    "d128_k512_cluster4": ([300, 1, 513], 2, 128, 512, None),
    "d128_k1024_cluster8": ([257, 90], 1, 128, 1024, None),
    "d64_k16": ([1000, 5], 1, 64, 16, None),
    "d128_k192_kc96": ([400, 77], 2, 128, 192, None),
    "d64_k96": ([333], 3, 64, 96, None),
    "d128_k128_long_chains": ([6000, 2100], 1, 128, 128, None),
}


@pytest.mark.parametrize("name", sorted(MASS_CASES))
def test_proto_mass_parity(name):
    """mass[b,h,j] = sum_i A[j,i] (Eq. (8)): element-wise against the oracle, and summed over the
    prototypes it is the user's valid length."""
    lengths, H, d, k, su = MASS_CASES[name]
    inp = W.make_sa(lengths, H, d, k, seed=600 + len(name), seqused=su)
    sk, lse, ms = run_gpu(inp, mass=True)
    osk, olse, oms = run_oracle(inp)
    assert_close(sk, osk, "sketch")
    assert_close(lse, olse, "lse")
    assert_close(ms, oms, "mass")
    _conservation(inp, sk, ms)
    # the mass plan (at most 128 prototypes per CTA) gives the same sketch within tolerance
    sk2, lse2 = run_gpu(inp)
    assert np.abs(sk2 - sk).max() < 5e-3 and np.array_equal(lse2 == -np.inf, lse == -np.inf)


def test_proto_mass_deterministic():
    inp = W.make_sa([3000, 1700], 2, 128, 512, seed=61)
    a = run_gpu(inp, mass=True)
    b = run_gpu(inp, mass=True)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("d,k", [(64, 256), (128, 512), (128, 64)])
def test_proto_keys_alias_values(d, k):
    """k and v the same device tensor: the paper's V = X (Eq. (9))."""
    inp = W.make_sa([700, 129, 1], 2, d, k, seed=62 + d + k)
    sk, lse = run_gpu(inp, alias=True)
    osk, olse, _ = run_oracle(inp, alias=True)
    assert_close(sk, osk, "sketch (k is v)")
    assert_close(lse, olse, "lse (k is v)")


def test_proto_large_values_with_small_weights():
    """|v| up to 1e5 (beyond fp16) is exact enough when every weight times the value stays in
    range: the values are scaled per token by the token's largest weight before fp16."""
    inp = W.make_sa([900, 300], 2, 128, 512, seed=63)
    s = 3.0e4
    v = (inp.v.float() * s).bfloat16()
    big = W.SAInputs(inp.q, inp.k, v, inp.cu_seqlens, None, inp.scale, inp.norm)
    assert float(v.float().abs().max()) > 65504
    sk, lse, st = run_gpu(big, status=True)
    osk, olse, _ = run_oracle(big)
    assert st == 0
    assert_close(sk, osk, "sketch (|v| > 65504)", scale=s)
    assert_close(lse, olse, "lse")


def test_proto_weighted_overflow_is_reported():
    """A token whose weight on one prototype is ~1 and whose value row exceeds the fp16 range:
    the call records SKA_ERR_RANGE and the affected sketch entries are not finite."""
    inp = W.make_sa([200, 150], 1, 64, 16, seed=64)
    q = inp.q.float()
    k = inp.k.float().clone()
    v = inp.v.float().clone()
    k[5, 0] = q[0, 3] / q[0, 3].norm() * 60.0  # token 5 of user 0 puts ~all its weight on prototype 3
    v[5, 0] = 1.0e5
    bad = W.SAInputs(inp.q, k.bfloat16(), v.bfloat16(), inp.cu_seqlens, None, inp.scale, inp.norm)
    sk, lse, st = run_gpu(bad, status=True)
    assert st == 6  # SKA_ERR_RANGE
    assert not np.isfinite(sk[0, 0]).all()


def test_timeout_is_reported_not_hung():
    """A withheld producer arrival makes the consumers' bounded waits run out; the kernel
    records SKA_ERR_DEVICE_TIMEOUT and exits, and the context stays usable."""
    api = _api()
    inp = W.make_sa([600, 300], 2, 128, 512, seed=15)
    dev = "cuda"
    ws = torch.zeros(api.sa_forward_workspace_size(api.sa_desc(inp.q, inp.k, inp.cu_seqlens, scale=1.0,
                                                               norm="proto")), dtype=torch.uint8, device=dev)
    try:
        api.set_debug(50_000_000, 1)
        api.sa_forward(inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), inp.cu_seqlens.to(dev), workspace=ws)
        st = api.read_device_status(ws)
    finally:
        api.set_debug(0, 0)
    assert st == 5  # SKA_ERR_DEVICE_TIMEOUT
    check_proto(inp)  # the next call on the same context is correct
