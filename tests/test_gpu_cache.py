"""GPU parity of the sketch cache (SequenceO1 §4.1) against its oracle model: the same sequence of
put and get batches gives the same slots, hits and rows, bit for bit. The keys are drawn from a
small pool, so that sets are shared within batches. The times advance past the TTL, so that
expiry, refresh and eviction all happen."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def _api():
    from sketch_attention_flashsa_b200 import api
    return api


def _keys(pool, idx):
    return [pool[i] for i in idx]


@pytest.mark.parametrize("num_sets,ways,ttl", [(16, 4, 30), (64, 8, 1000), (1, 32, 5), (4096, 1, 20)])
def test_cache_matches_model(num_sets, ways, ttl):
    api = _api()
    rng = np.random.default_rng(num_sets + ways)
    row = 12
    pool = [(int(rng.integers(0, 2**63)), int(rng.integers(0, 3)), int(rng.integers(0, 2)), int(rng.integers(0, 5)))
            for _ in range(200)]
    model = oracle.SketchCache(num_sets, ways, row, ttl)
    cache = api.SketchCache(num_sets, ways, row, ttl)

    def dev_keys(ks):
        return api.cache_keys([k[0] for k in ks], [k[1] for k in ks], [k[2] for k in ks], [k[3] for k in ks])

    now = 0
    for step in range(40):
        now += int(rng.integers(0, 4))
        n = int(rng.integers(1, 120))
        ks = _keys(pool, rng.integers(0, len(pool), n))
        if step % 2 == 0:
            rows = rng.standard_normal((n, row)).astype(np.float32)
            slots = cache.put(dev_keys(ks), torch.from_numpy(rows).cuda(), now)
            want = model.put(ks, rows.astype(np.float64), now)
            torch.cuda.synchronize()
            assert slots.cpu().tolist() == want, step
        else:
            out, hits = cache.get(dev_keys(ks), now)
            whits, wrows = model.get(ks, now)
            torch.cuda.synchronize()
            assert hits.cpu().numpy().astype(bool).tolist() == whits.tolist(), step
            assert np.array_equal(out.cpu().numpy().astype(np.float64), wrows), step


def test_cache_round_trip_of_a_sketch():
    """A batch of SA sketches [B, H, k, d] stored per user and read back whole."""
    api = _api()
    B, H, k, d = 6, 2, 64, 64
    sk = torch.randn(B, H * k * d, device="cuda")
    cache = api.SketchCache(256, 4, H * k * d, 3600)
    keys = api.cache_keys(list(range(100, 100 + B)), 7, 1, 1_700_000_000)
    cache.put(keys, sk, 0)
    out, hits = cache.get(keys, 3600)
    torch.cuda.synchronize()
    assert hits.all() and torch.equal(out, sk)
    out, hits = cache.get(keys, 3601)            # past the TTL
    torch.cuda.synchronize()
    assert not hits.any() and not out.any()
