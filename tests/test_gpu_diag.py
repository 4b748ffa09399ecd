"""GPU parity of the allocation diagnostics against the fp64 oracle:
- each token's largest prototype-wise weight, the Fig. 3 quantity of SequenceO1 §5.1;
- its histogram;
- the mass-renormalised (Slot-Attention weighted-mean) sketch, §2.4.

The weights come out of the fp32 softmax, so they are held to the SA bar: max abs ≤ 1e-2,
rel-L2 ≤ 5e-3. The histogram is compared with the oracle's histogram of the GPU's own max weights,
bit-exact. That is an integer decision taken on the same fp32 values. Against the oracle's own max
weights it only has to agree to within the values that sit at bin edges."""
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


CASES = {
    "d64_k256_ragged_padded": ([700, 129, 1, 300], 2, 64, 256, [650, 129, 1, 40]),
    "d128_k512_cluster2": ([300, 513], 2, 128, 512, None),
    "d128_k128": ([1000, 7], 1, 128, 128, [1000, 0]),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_max_weight_histogram_and_renormalised_sketch(name):
    lengths, H, d, k, su = CASES[name]
    inp = W.make_sa(lengths, H, d, k, seed=800 + len(name), seqused=su)
    api = _api()
    g = lambda t: None if t is None else t.cuda()  # noqa: E731
    sk, lse, mass, mw = api.sa_forward_diag(g(inp.q), g(inp.k), g(inp.v), g(inp.cu_seqlens), g(inp.seqused),
                                            scale=inp.scale, renormalize=True)
    counts = api.weight_histogram(mw, 20)
    torch.cuda.synchronize()
    sun = inp.seqused.numpy() if inp.seqused is not None else None
    o_sk, _, o_mass = oracle.sa_forward(f64(inp.q), f64(inp.k), f64(inp.v), inp.cu_seqlens.numpy(), sun, inp.scale, 0)
    o_mw = oracle.token_max_weight(f64(inp.q), f64(inp.k), f64(inp.v), inp.cu_seqlens.numpy(), sun, inp.scale)
    gm = mw.cpu().numpy().astype(np.float64)
    assert (gm[o_mw < 0] == -1).all(), "padding rows carry -1"
    assert_close(gm[o_mw >= 0], o_mw[o_mw >= 0], "max weight")
    assert (gm[o_mw >= 0] >= 1.0 / k - 1e-6).all() and (gm[o_mw >= 0] <= 1 + 1e-6).all()
    assert_close(mass.cpu().numpy().astype(np.float64), o_mass, "mass")
    assert_close(sk.cpu().numpy().astype(np.float64), oracle.renormalized_sketch(o_sk, o_mass), "renormalised sketch")
    c = counts.cpu().numpy()
    assert np.array_equal(c, oracle.weight_histogram(gm, 20)), "histogram of the same values"
    assert c.sum() == (o_mw >= 0).sum()
    # the oracle's own maxima fall into the same bins except where a value sits within 1e-3 of an edge
    o_c = oracle.weight_histogram(o_mw, 20)
    near = np.abs((o_mw[o_mw >= 0] * 20) - np.round(o_mw[o_mw >= 0] * 20)) < 2e-2
    assert np.abs(c - o_c).sum() <= 2 * near.sum()


def test_diag_without_renormalisation_matches_sa_forward_bitwise():
    inp = W.make_sa([900, 40], 2, 128, 256, seed=83)
    api = _api()
    g = lambda t: t.cuda()  # noqa: E731
    sk, lse, mass, mw = api.sa_forward_diag(g(inp.q), g(inp.k), g(inp.v), g(inp.cu_seqlens), scale=inp.scale)
    sk2, lse2, mass2 = api.sa_forward(g(inp.q), g(inp.k), g(inp.v), g(inp.cu_seqlens), scale=inp.scale,
                                      want_mass=True)
    torch.cuda.synchronize()
    assert torch.equal(sk, sk2) and torch.equal(lse, lse2) and torch.equal(mass, mass2)


def test_histogram_exact_counts():
    api = _api()
    vals = torch.tensor([0.0, 0.1, 0.5, 0.999, 1.0, 0.25, -1.0, float("nan")] * 1000, device="cuda")
    c = api.weight_histogram(vals, 4)
    torch.cuda.synchronize()
    assert c.cpu().tolist() == [2000, 1000, 1000, 2000]
