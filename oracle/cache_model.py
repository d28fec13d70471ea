"""Plain host model of the prefix-hash block cache (test infrastructure only).

MapFlow page "MapFlow开源:大模型换班,Prefill为何能快20%?" (aitest123.com), section
"存不下、读得慢?三个工程优化手段", subsection 2 "找得快的:基于前缀哈希的缓存管理", and its English
rendering (roboind.com, section "When it comes to real savings in reuse..."): the kept blocks,
whose number differs per layer and position, are indexed by a prefix hash that carries the
preceding context, and a receiver finds its blocks through that index.

Readings taken where the pages are silent (the same ones the library documents):
  - the hash of query block k is 64-bit FNV-1a of the little-endian bytes of every token up
    to the end of that block, so equal hashes mean equal preceding context;
  - an entry is one query-block row of one sender layer, keyed by (layer, hash): its kept
    key-block indices and the values of those blocks;
  - a request reuses the longest cached prefix of its rows: the walk stops at the first row
    that is not cached (one miss) or whose blocks no longer fit the output (no miss);
  - the pool holds a fixed number of block slots; a row that is inserted takes one slot per
    kept block; rows are evicted least recently used first (a put or a hit makes a row the
    most recent); a row already cached is only made the most recent; a row larger than the
    pool, or one that reaches past the capacity of the compressed layer it comes from (an
    overflowed compression did not write all its blocks), is not cached.

Nothing here is shared with the CUDA library: this is an independent statement of what the
cache must return, in ordinary Python containers, written for reading rather than speed.
"""
from collections import OrderedDict

import numpy as np

FNV_OFFSET_BASIS = 0xcbf29ce484222325
FNV_PRIME = 0x100000001b3  # 2^40 + 2^8 + 0xb3
_MASK = (1 << 64) - 1


def fnv1a64(data: bytes, h: int = FNV_OFFSET_BASIS) -> int:
    """FNV-1a, 64 bits (Fowler, Noll, Vo): for each byte, xor it in, then multiply by the prime."""
    for byte in data:
        h = ((h ^ byte) * FNV_PRIME) & _MASK
    return h


def prefix_hashes(tokens, B):
    """Hash of every query block: FNV-1a 64 of the int32 little-endian bytes of tokens[0 .. end
    of the block), continued across blocks so each value covers the whole prefix."""
    toks = np.asarray(tokens, dtype=np.int32)
    out, h = [], FNV_OFFSET_BASIS
    for k in range(-(-len(toks) // B)):
        h = fnv1a64(toks[k * B:(k + 1) * B].astype("<i4").tobytes(), h)
        out.append(h)
    return out


class PrefixCacheModel:
    """The cache's bookkeeping and contents, one Python object per cached row."""

    def __init__(self, n_slots):
        self.n_slots = n_slots
        self.free = n_slots
        # (layer, hash) -> (kept key blocks, their values); first = least recently used
        self.rows = OrderedDict()
        self.hits = self.misses = self.evicted = 0

    def put(self, layer, row_ptr, col_idx, values, capacity, row0, hashes):
        """Insert rows row0 .. row0 + len(hashes) - 1 of a compressed layer (row_ptr, col_idx,
        values: host copies of its BSR; capacity: its capacity in blocks).  Returns the number
        of rows inserted."""
        inserted = 0
        for r, h in enumerate(hashes):
            key = (layer, int(h))
            if key in self.rows:
                self.rows.move_to_end(key)
                continue
            b0, b1 = int(row_ptr[row0 + r]), int(row_ptr[row0 + r + 1])
            if b1 > capacity:
                continue
            need = b1 - b0
            if need <= 0 or need > self.n_slots:
                continue
            while self.free < need and self.rows:
                _, (cols, _) = self.rows.popitem(last=False)
                self.free += len(cols)
                self.evicted += 1
            self.rows[key] = (list(map(int, col_idx[b0:b1])), np.array(values[b0:b1]))
            self.free -= need
            inserted += 1
        return inserted

    def get(self, layer, hashes, capacity):
        """Assemble the longest cached prefix of a request's rows.  Returns (rows found,
        row_ptr [found + 1], col_idx [n], values [n, ...])."""
        row_ptr, cols, vals = [0], [], []
        found = 0
        for h in hashes:
            key = (layer, int(h))
            if key not in self.rows:
                self.misses += 1
                break
            c, v = self.rows[key]
            if row_ptr[-1] + len(c) > capacity:
                break
            cols.extend(c)
            vals.append(v)
            row_ptr.append(row_ptr[-1] + len(c))
            self.rows.move_to_end(key)
            self.hits += 1
            found += 1
        values = np.concatenate(vals) if vals else None
        return found, row_ptr, cols, values

    def stats(self):
        """rows, used slots, free slots, hits, misses, evictions."""
        return {"rows": len(self.rows), "used": self.n_slots - self.free, "free": self.free,
                "hits": self.hits, "misses": self.misses, "evicted": self.evicted}

    def cached(self, layer):
        """Hashes of the layer's cached rows, least recently used first."""
        return [h for (l, h) in self.rows if l == layer]
