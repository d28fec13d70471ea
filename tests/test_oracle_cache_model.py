"""Pins of the host model of the prefix-hash block cache (oracle/cache_model.py).

- FNV-1a 64 against the published test vectors of its authors (Fowler, Noll, Vo).
- The prefix property of the block hashes: block k's hash is the hash of the whole prefix.
- A hand-worked sequence of puts and gets: slot accounting, LRU eviction order, the prefix walk
  stopping at a miss or at the output capacity, rows refused for size or an overflowed source.
- Random operation sequences against a second, timestamp-based formulation of the same rules
  (least recently used = smallest last-use time), so a slip in the ordered-dict bookkeeping
  (a missed refresh, the wrong end evicted) shows up as a disagreement.
"""
import numpy as np
import pytest

from oracle.cache_model import PrefixCacheModel, fnv1a64, prefix_hashes


def test_fnv1a64_published_vectors():
    assert fnv1a64(b"") == 0xcbf29ce484222325
    assert fnv1a64(b"a") == 0xaf63dc4c8601ec8c
    assert fnv1a64(b"foobar") == 0x85944171f73967e8


def test_prefix_hashes_cover_the_whole_prefix():
    toks = np.array([5, -1, 70000, 3, 9, 11, 2], dtype=np.int32)
    h = prefix_hashes(toks, 3)
    assert len(h) == 3
    for k in range(3):
        assert h[k] == fnv1a64(toks[:min(3 * (k + 1), len(toks))].astype("<i4").tobytes())
    assert prefix_hashes(np.zeros(0, np.int32), 3) == []


def _bsr(sizes, h_s=1, B=2):
    """A toy compressed layer: row r has sizes[r] blocks whose values are filled with 100 r + k."""
    row_ptr = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    col_idx = np.concatenate([np.arange(n) for n in sizes]).astype(np.int32)
    values = np.zeros((row_ptr[-1], h_s, B, B), dtype=np.float32)
    for r, n in enumerate(sizes):
        for k in range(n):
            values[row_ptr[r] + k] = 100 * r + k
    return row_ptr, col_idx, values


def test_hand_worked_sequence():
    rp, ci, vals = _bsr([2, 2, 2, 6, 1])
    m = PrefixCacheModel(5)
    # rows 0, 1 in: 4 slots used
    assert m.put(0, rp, ci, vals, 100, 0, [10, 11]) == 2
    assert m.stats() == {"rows": 2, "used": 4, "free": 1, "hits": 0, "misses": 0, "evicted": 0}
    # a hit on row 0 makes it the most recent; row 1 is now least recently used
    found, rpo, cio, vo = m.get(0, [10], 100)
    assert found == 1 and rpo == [0, 2] and cio == [0, 1] and (vo[:, 0, 0, 0] == [0, 1]).all()
    # row 2 needs 2 slots, 1 is free: row 1 is evicted
    assert m.put(0, rp, ci, vals, 100, 2, [12]) == 1
    assert m.cached(0) == [10, 12] and m.stats()["evicted"] == 1
    # the prefix walk stops at the first miss (row 1) ...
    found, rpo, _, _ = m.get(0, [10, 11, 12], 100)
    assert found == 1 and rpo == [0, 2] and m.stats()["misses"] == 1
    # ... or where the output capacity runs out, without a miss
    found, rpo, _, _ = m.get(0, [10, 12], 3)
    assert found == 1 and m.stats()["misses"] == 1
    # another layer shares nothing
    assert m.get(1, [10], 100)[0] == 0
    # row 3 (6 blocks) is larger than the pool; row 4 reaches past a capacity of 8: refused
    assert m.put(0, rp, ci, vals, 100, 3, [13]) == 0
    assert m.put(0, rp, ci, vals, 8, 4, [14]) == 0
    # a row already cached is only refreshed
    assert m.put(0, rp, ci, vals, 100, 0, [12]) == 0
    assert m.cached(0) == [10, 12]
    assert m.stats() == {"rows": 2, "used": 4, "free": 1, "hits": 3, "misses": 2, "evicted": 1}


class _TimestampModel:
    """The same rules with explicit last-use times (a second formulation for cross-checking)."""

    def __init__(self, n_slots):
        self.n_slots, self.t = n_slots, 0
        self.rows = {}  # key -> [last use, n blocks, first block index in the source]
        self.hits = self.misses = self.evicted = 0

    def _tick(self):
        self.t += 1
        return self.t

    def used(self):
        return sum(v[1] for v in self.rows.values())

    def put(self, layer, rp, capacity, row0, hashes):
        ins = 0
        for r, h in enumerate(hashes):
            key = (layer, h)
            if key in self.rows:
                self.rows[key][0] = self._tick()
                continue
            b0, b1 = rp[row0 + r], rp[row0 + r + 1]
            if b1 > capacity or b1 - b0 <= 0 or b1 - b0 > self.n_slots:
                continue
            while self.n_slots - self.used() < b1 - b0 and self.rows:
                victim = min(self.rows, key=lambda k: self.rows[k][0])
                del self.rows[victim]
                self.evicted += 1
            self.rows[key] = [self._tick(), b1 - b0, b0]
            ins += 1
        return ins

    def get(self, layer, hashes, capacity):
        n = found = 0
        firsts = []
        for h in hashes:
            key = (layer, h)
            if key not in self.rows:
                self.misses += 1
                break
            if n + self.rows[key][1] > capacity:
                break
            n += self.rows[key][1]
            firsts.append(self.rows[key][2])
            self.rows[key][0] = self._tick()
            self.hits += 1
            found += 1
        return found, firsts


@pytest.mark.parametrize("seed", range(6))
def test_random_sequences_agree_with_timestamp_formulation(seed):
    rng = np.random.default_rng(seed)
    sizes = rng.integers(1, 6, size=40)
    rp, ci, vals = _bsr(sizes)
    n_slots = int(rng.integers(6, 30))
    a, b = PrefixCacheModel(n_slots), _TimestampModel(n_slots)
    hashes = list(range(1000, 1040))
    for _ in range(200):
        layer = int(rng.integers(0, 2))
        row0 = int(rng.integers(0, 38))
        n = int(rng.integers(1, 41 - row0))
        hs = hashes[row0:row0 + n]
        if rng.random() < 0.5:
            cap = int(rng.integers(rp[row0 + n - 1], rp[-1] + 1))
            assert a.put(layer, rp, ci, vals, cap, row0, hs) == b.put(layer, rp, cap, row0, hs)
        else:
            cap = int(rng.integers(0, 60))
            found, rpo, cio, vo = a.get(layer, hs, cap)
            found_b, firsts = b.get(layer, hs, cap)
            assert found == found_b
            # the assembled rows are the source rows named by the timestamp model
            want_cols = [c for f in firsts for c in ci[f:f + (rp[1:] - rp[:-1])[list(rp).index(f)]]]
            assert cio == want_cols
            if found:
                want_vals = np.concatenate([vals[f:f + (rp[1:] - rp[:-1])[list(rp).index(f)]] for f in firsts])
                assert (vo == want_vals).all()
        sa = a.stats()
        assert (sa["rows"], sa["used"], sa["hits"], sa["misses"], sa["evicted"]) == \
            (len(b.rows), b.used(), b.hits, b.misses, b.evicted)
