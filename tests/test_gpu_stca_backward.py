"""GPU parity of the STCA backward (SequenceO1 §2.3, §3.4; MRLB's per-target suffix lengths of
§4.2) against the fp64 oracle, through the C ABI. Same bar as the forward: max abs error <= 1e-2
and relative L2 <= 5e-3 on every gradient. The forward's out and lse that the backward consumes
come from the GPU forward, as in training; the oracle recomputes its own."""
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


def run_gpu(inp: W.STCAInputs, status=False):
    api = _api()
    g = lambda t: None if t is None else t.cuda()  # noqa: E731
    ks = inp.k_sk.shape[2]
    k_sk, v_sk = (g(inp.k_sk), g(inp.v_sk)) if ks > 0 else (None, None)
    kvl = g(inp.target_kv_len)
    out, lse = api.stca_forward(g(inp.q), g(inp.cu_targets), g(inp.k_hist), g(inp.v_hist), g(inp.cu_hist), k_sk,
                                v_sk, scale=inp.scale, target_kv_len=kvl)
    desc = api.stca_desc(inp.q, inp.k_hist, k_sk, inp.cu_targets, inp.cu_hist, scale=inp.scale, max_targets=1)
    ws = torch.empty(max(int(api._lib.lib().stca_backward_workspace_size(__import__("ctypes").byref(desc))), 256),
                     dtype=torch.uint8, device="cuda")
    grads = api.stca_backward(g(inp.q), g(inp.cu_targets), g(inp.k_hist), g(inp.v_hist), g(inp.cu_hist), k_sk, v_sk,
                              out, lse, g(inp.dout), scale=inp.scale, target_kv_len=kvl, workspace=ws)
    torch.cuda.synchronize()
    res = [None if t is None else t.cpu().numpy().astype(np.float64) for t in grads]
    if status:
        res.append(api.read_device_status(ws))
    return res


def run_oracle(inp: W.STCAInputs):
    kvl = inp.target_kv_len.numpy() if inp.target_kv_len is not None else None
    return oracle.stca_backward(f64(inp.q), inp.cu_targets.numpy(), f64(inp.k_hist), f64(inp.v_hist),
                                inp.cu_hist.numpy(), f64(inp.k_sk), f64(inp.v_sk), inp.scale, f64(inp.dout), kvl)


NAMES = ("dq", "dk_hist", "dv_hist", "dk_sk", "dv_sk")


def check(inp):
    got = run_gpu(inp, status=True)
    assert got[-1] == 0
    want = run_oracle(inp)
    for name, g, w in zip(NAMES, got[:5], want):
        if w.size == 0:
            continue
        assert_close(g, w, name)
    return got


CASES = {
    # (targets per user, suffix per user, heads, d, sketch rows, kv lengths)
    "d64_ragged": ([3, 130, 1], [200, 5, 129], 2, 64, 40, False),
    "d128_ragged_kvlen": ([70, 260], [300, 131], 2, 128, 130, True),
    "d64_no_sketch": ([129, 2], [256, 77], 1, 64, 0, False),
    "d64_kvlen_many_tiles": ([300], [1100], 2, 64, 256, True),
    "d128_one_target": ([1, 1, 1], [1, 400, 0], 1, 128, 3, False),
    # a user with no targets (its keys get zero gradients) and one with no suffix
    "d64_empty_users": ([0, 50, 20], [90, 0, 33], 2, 64, 17, True),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_stca_backward_parity(name):
    targets, hist, H, d, ks, kvl = CASES[name]
    inp = W.make_stca(targets, hist, H, d, ks, seed=600 + len(name), with_kv_len=kvl, with_dout=True)
    got = check(inp)
    if name == "d64_empty_users":
        # user 0 has no targets: its suffix rows (0..89) get exactly zero
        assert not got[1][:90].any() and not got[2][:90].any()


def test_stca_backward_long_chains():
    """2,300 suffix keys: 18 key tiles, so dq sums two TMEM chains per target tile."""
    inp = W.make_stca([200], [2300], 1, 64, 64, seed=611, with_dout=True)
    check(inp)


def test_stca_backward_deterministic():
    inp = W.make_stca([150, 40], [500, 260], 2, 64, 32, seed=612, with_kv_len=True, with_dout=True)
    a = run_gpu(inp)
    b = run_gpu(inp)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_stca_backward_config5_two_users():
    """Config 5 (16 users x 512 targets, 10,000 suffix + 256 sketch keys, H = 4, d = 64, scale 1/8)
    through the GPU in full; users 0 and 15 compared with the oracle element by element (every
    gradient of a user depends on that user's inputs only)."""
    cfg = W.config5()
    rng = np.random.default_rng(4)  # upstream gradient for the full batch
    inp = W.STCAInputs(cfg.q, cfg.cu_targets, cfg.k_hist, cfg.v_hist, cfg.cu_hist, cfg.k_sk, cfg.v_sk, cfg.scale,
                       None, W.to_bf16(W.normal(rng, tuple(cfg.q.shape))))
    got = run_gpu(inp, status=True)
    assert got[-1] == 0
    for b in (0, 15):
        t0, t1 = int(cfg.cu_targets[b]), int(cfg.cu_targets[b + 1])
        h0, h1 = int(cfg.cu_hist[b]), int(cfg.cu_hist[b + 1])
        sub = W.STCAInputs(cfg.q[t0:t1], torch.tensor([0, t1 - t0], dtype=torch.int32), cfg.k_hist[h0:h1],
                           cfg.v_hist[h0:h1], torch.tensor([0, h1 - h0], dtype=torch.int32), cfg.k_sk[b:b + 1],
                           cfg.v_sk[b:b + 1], cfg.scale, None, inp.dout[t0:t1])
        want = run_oracle(sub)
        assert_close(got[0][t0:t1], want[0], f"user {b} dq")
        assert_close(got[1][h0:h1], want[1], f"user {b} dk_hist")
        assert_close(got[2][h0:h1], want[2], f"user {b} dv_hist")
        assert_close(got[3][b:b + 1], want[3], f"user {b} dk_sk")
        assert_close(got[4][b:b + 1], want[4], f"user {b} dv_sk")
