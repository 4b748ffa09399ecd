"""GPU parity of the SA backward (libska.so through its C ABI) against the fp64 oracle, both
normalisations. Tolerance as for the forward: max abs error <= 1e-2 and relative L2 <= 5e-3 on
dQ, dK and dV. The forward outputs fed to the backward (lse, and the sketch for the token-wise
D_j term) come from the oracle, so a forward error cannot hide or cause a backward one."""
import numpy as np
import pytest
import torch

import oracle
from sketch_attention_flashsa_b200 import workloads as W

from test_gpu_sa_forward import assert_close, f64

pytestmark = pytest.mark.gpu


def _api():
    from sketch_attention_flashsa_b200 import api
    return api


def run_bwd(inp: W.SAInputs, norm: str, osk, olse):
    api = _api()
    dev = "cuda"
    su = inp.seqused.to(dev) if inp.seqused is not None else None
    lse = torch.from_numpy(olse.astype(np.float32)).to(dev)
    sk = torch.from_numpy(osk.astype(np.float32)).to(dev)
    dq, dk, dv = api.sa_backward(inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), inp.cu_seqlens.to(dev), su, lse,
                                 inp.dsketch.to(dev), sk, scale=inp.scale, norm=norm)
    torch.cuda.synchronize()
    return [x.cpu().numpy().astype(np.float64) for x in (dq, dk, dv)]


def check_bwd(inp: W.SAInputs, norm: str):
    nid = W.NORM_PROTO if norm == "proto" else W.NORM_TOKEN
    su = inp.seqused.numpy() if inp.seqused is not None else None
    osk, olse, _ = oracle.sa_forward(f64(inp.q), f64(inp.k), f64(inp.v), inp.cu_seqlens.numpy(), su, inp.scale, nid)
    dq, dk, dv = run_bwd(inp, norm, osk, olse)
    odq, odk, odv = oracle.sa_backward(f64(inp.q), f64(inp.k), f64(inp.v), inp.cu_seqlens.numpy(), su,
                                       f64(inp.dsketch), inp.scale, nid)
    assert_close(dq, odq, f"{norm} dq")
    assert_close(dk, odk, f"{norm} dk")
    assert_close(dv, odv, f"{norm} dv")
    return dq, dk, dv


CASES = {
    "d64_k256_ragged": ([1, 127, 128, 129, 700], 2, 64, 256),
    "d64_k16": ([300, 5], 1, 64, 16),
    "d128_k128": ([400, 129], 2, 128, 128),
    "d64_k64": ([257], 3, 64, 64),
}


@pytest.mark.parametrize("norm", ["proto", "token"])
@pytest.mark.parametrize("name", sorted(CASES))
def test_backward_parity_small(name, norm):
    lengths, H, d, k = CASES[name]
    inp = W.make_sa(lengths, H, d, k, seed=500 + len(name), with_dsketch=True, dsketch_seed=7)
    check_bwd(inp, norm)


# More prototypes than one CTA holds: one launch per chunk of 128 (d = 128) or 256 (d = 64)
# prototypes, PROTO's delta_i summed over the chunks by a first pass.
CHUNK_CASES = {
    "d128_k256": ([1, 127, 129, 600], 2, 128, 256),
    "d128_k384": ([250, 3], 1, 128, 384),
    "d128_k512": ([300, 0, 517], 2, 128, 512),
    "d64_k512": ([700, 129], 2, 64, 512),
    "d64_k1024": ([400], 1, 64, 1024),
}


@pytest.mark.parametrize("norm", ["proto", "token"])
@pytest.mark.parametrize("name", sorted(CHUNK_CASES))
def test_backward_parity_prototype_chunks(name, norm):
    lengths, H, d, k = CHUNK_CASES[name]
    inp = W.make_sa(lengths, H, d, k, seed=540 + len(name) + k, with_dsketch=True, dsketch_seed=17)
    check_bwd(inp, norm)


@pytest.mark.parametrize("norm", ["proto", "token"])
def test_backward_prototype_chunks_padding_per_user(norm):
    inp = W.make_sa([200, 0, 300, 130], 2, 128, 512, seed=57, seqused=[150, 0, 1, 130], per_user_q=True,
                    with_dsketch=True, dsketch_seed=18)
    dq, dk, dv = check_bwd(inp, norm)
    assert (dk[150:200] == 0).all() and (dv[150:200] == 0).all()
    assert (dk[201:500] == 0).all() and (dv[201:500] == 0).all()


@pytest.mark.parametrize("norm", ["proto", "token"])
def test_backward_prototype_chunks_deterministic(norm):
    inp = W.make_sa([3000, 1700], 2, 128, 512, seed=58, with_dsketch=True, dsketch_seed=19)
    nid = W.NORM_PROTO if norm == "proto" else W.NORM_TOKEN
    osk, olse, _ = oracle.sa_forward(f64(inp.q), f64(inp.k), f64(inp.v), inp.cu_seqlens.numpy(), None, 1.0, nid)
    a = run_bwd(inp, norm, osk, olse)
    b = run_bwd(inp, norm, osk, olse)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("norm", ["proto", "token"])
def test_backward_padding_empty_per_user(norm):
    inp = W.make_sa([200, 0, 300, 130], 2, 64, 256, seed=51, seqused=[150, 0, 1, 130], per_user_q=True,
                    with_dsketch=True, dsketch_seed=8)
    dq, dk, dv = check_bwd(inp, norm)
    assert (dk[150:200] == 0).all() and (dv[150:200] == 0).all()
    assert (dk[201:500] == 0).all() and (dv[201:500] == 0).all()


@pytest.mark.parametrize("norm", ["proto", "token"])
def test_backward_deterministic(norm):
    inp = W.make_sa([3000, 1700], 2, 64, 256, seed=52, with_dsketch=True, dsketch_seed=9)
    nid = W.NORM_PROTO if norm == "proto" else W.NORM_TOKEN
    osk, olse, _ = oracle.sa_forward(f64(inp.q), f64(inp.k), f64(inp.v), inp.cu_seqlens.numpy(), None, 1.0, nid)
    a = run_bwd(inp, norm, osk, olse)
    b = run_bwd(inp, norm, osk, olse)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("norm", ["proto", "token"])
def test_backward_long_chains(norm):
    """240K tokens x 2 heads = 3752 tiles over the SMs: every CTA walks dozens of tiles of one
    (user, head), so dQ is restarted and added into its partial slot several times."""
    inp = W.make_sa([150_000, 90_000], 2, 64, 128, seed=53, with_dsketch=True, dsketch_seed=10)
    check_bwd(inp, norm)


@pytest.mark.slow
@pytest.mark.parametrize("norm", ["proto", "token"])
def test_backward_config4_full(norm):
    """Config 4: config-2 shapes (64 ragged users up to 91K tokens, H=4, d=64, k=256), dQ reduced
    over all 1.45M tokens; dQ, dK and dV of every user compared with the oracle."""
    inp = W.config4(W.NORM_PROTO if norm == "proto" else W.NORM_TOKEN)
    nid = inp.norm
    cu = inp.cu_seqlens.numpy()
    q, k, v, do = f64(inp.q), inp.k, inp.v, f64(inp.dsketch)
    B, H = inp.num_users, inp.num_heads
    osk = np.zeros((B, H, inp.num_protos, inp.head_dim))
    olse = np.full((inp.total_tokens, H), -np.inf) if nid == W.NORM_PROTO else np.zeros((B, H, inp.num_protos))
    for b in range(B):
        lo, hi = int(cu[b]), int(cu[b + 1])
        kb, vb = f64(k[lo:hi]), f64(v[lo:hi])
        for h in range(H):
            sk, ls, _, _ = oracle.sa_problem(q[h], kb[:, h], vb[:, h], inp.scale, nid)
            osk[b, h] = sk
            if nid == W.NORM_PROTO:
                olse[lo:hi, h] = ls
            else:
                olse[b, h] = ls
    dq, dk, dv = run_bwd(inp, norm, osk, olse)
    odq = np.zeros_like(q)
    worst = 0.0
    for b in range(B):
        lo, hi = int(cu[b]), int(cu[b + 1])
        gq, gk, gv = oracle.sa_backward(q, f64(k[lo:hi]), f64(v[lo:hi]), np.array([0, hi - lo]), None, do[b:b + 1],
                                        inp.scale, nid)
        odq += gq
        mk, _ = assert_close(dk[lo:hi], gk, f"{norm} dk user {b}")
        mv, _ = assert_close(dv[lo:hi], gv, f"{norm} dv user {b}")
        worst = max(worst, mk, mv)
    assert_close(dq, odq, f"{norm} dq (all users)")
    print(f"[parity] dK, dV of all {B} users, worst max abs {worst:.3e}")


@pytest.mark.slow
@pytest.mark.parametrize("norm", ["proto", "token"])
def test_backward_production_shape_k1024(norm):
    """App. G.5's shapes (d = 128, k up to 1024): 6 ragged users up to 24K tokens, H = 2,
    k = 1024 (eight chunks of 128 prototypes); dQ, dK and dV of every user against the oracle."""
    inp = W.make_sa([24_000, 9_001, 1, 16_384, 130, 20_000], 2, 128, 1024, seed=59, with_dsketch=True,
                    dsketch_seed=20)
    check_bwd(inp, norm)
