"""Model of the sketch cache of SequenceO1 §4.1, the contract the device cache must meet exactly.

TEST INFRASTRUCTURE ONLY (see the package docstring).

What the page specifies (§4.1 "Training-Side Local KVCache and Serving Reuse"):
- the cache holds the user-only sketch X~_u (k x d per head) because it is target-agnostic;
- an entry's key is (user id, model version, history timestamp, sketch configuration);
- entries are invalidated by a TTL, and capacity eviction bounds the memory;
- training and serving share one get/put interface.

Readings taken here, where the page gives no mechanism:
* The cache has S sets (a power of two) of W ways. A key's set is SplitMix64 applied in turn to the
  user id, version, configuration and timestamp (each folded in by xor), masked to S - 1.
  SplitMix64 follows its published definition (Steele, Lea and Flood, 2014; Vigna's reference code):
  z = x + 0x9E3779B97F4A7C15, then the xor-shift-multiply mix.
* get(keys, now): a key hits when a way of its set holds the same key, stored at time t with
  now - t <= ttl. A hit returns the stored sketch.
* put(keys, sketches, now): keys are applied in batch order. A way holding the same key is
  overwritten. Otherwise the first way that is empty or expired (now - t > ttl) takes the key, and
  failing that the way with the oldest time (ties: the lowest way). The stored time becomes now.
"""
from __future__ import annotations

import numpy as np

MASK = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15


def splitmix64(x: int) -> int:
    """One SplitMix64 step from state x: the output for state x + golden gamma."""
    z = (x + GOLDEN) & MASK
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK
    return z ^ (z >> 31)


def key_hash(user: int, version: int, config: int, timestamp: int) -> int:
    h = splitmix64(user & MASK)
    h = splitmix64(h ^ (version & 0xFFFFFFFF))
    h = splitmix64(h ^ (config & 0xFFFFFFFF))
    return splitmix64(h ^ (timestamp & MASK))


class SketchCache:
    def __init__(self, num_sets: int, ways: int, row: int, ttl: int):
        assert num_sets & (num_sets - 1) == 0
        self.S, self.W, self.row, self.ttl = num_sets, ways, row, ttl
        self.keys = [[None] * ways for _ in range(num_sets)]
        self.stamp = [[None] * ways for _ in range(num_sets)]
        self.data = np.zeros((num_sets, ways, row))

    def set_of(self, key) -> int:
        return key_hash(*key) & (self.S - 1)

    def _live(self, s, w, now) -> bool:
        return self.stamp[s][w] is not None and now - self.stamp[s][w] <= self.ttl

    def get(self, keys, now):
        """keys: list of (user, version, config, timestamp). Returns (hits [n] bool, rows [n, row])."""
        hits = np.zeros(len(keys), dtype=bool)
        rows = np.zeros((len(keys), self.row))
        for i, key in enumerate(keys):
            s = self.set_of(key)
            for w in range(self.W):
                if self.keys[s][w] == tuple(key) and self._live(s, w, now):
                    hits[i] = True
                    rows[i] = self.data[s, w]
                    break
        return hits, rows

    def put(self, keys, rows, now):
        """Applies the keys in batch order; returns the slot (set * W + way) each key was written to."""
        slots = []
        for i, key in enumerate(keys):
            key = tuple(key)
            s = self.set_of(key)
            way = next((w for w in range(self.W) if self.keys[s][w] == key), None)
            if way is None:
                way = next((w for w in range(self.W) if not self._live(s, w, now)), None)
            if way is None:
                way = min(range(self.W), key=lambda w: (self.stamp[s][w], w))
            self.keys[s][way] = key
            self.stamp[s][way] = now
            self.data[s, way] = rows[i]
            slots.append(s * self.W + way)
        return slots
