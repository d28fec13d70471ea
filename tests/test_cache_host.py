"""Host side of the prefix-hash block cache (no GPU): prefix hashes and cache bookkeeping.

The hash is 64-bit FNV-1a (Fowler-Noll-Vo; offset basis 0xcbf29ce484222325, prime 2^40 + 2^8 +
0xb3) over the little-endian bytes of the whole prefix up to the end of each query block
(MapFlow page "MapFlow开源:大模型换班,Prefill为何能快20%?", section "存不下、读得慢?三个工程
优化手段", subsection 2: a prefix hash carrying the preceding context)."""
import ctypes

import numpy as np
import pytest

from oracle.cache_model import prefix_hashes


@pytest.fixture(scope="module")
def mf():
    import __graft_entry__
    __graft_entry__.load_builder().build()
    import cross_model_attention_mf_b200 as mf
    return mf


def test_prefix_hashes_definition_and_prefix_property(mf):
    rng = np.random.default_rng(0)
    toks = rng.integers(-5, 150000, size=333).astype(np.int32)
    h = mf.mf_prefix_hashes(toks, 64)
    assert h.tolist() == prefix_hashes(toks, 64)  # the oracle's FNV-1a, pinned to published vectors
    assert len(h) == 6
    # a shared prefix gives shared hashes up to the first differing block, then none
    other = toks.copy()
    other[200] += 1                      # block 3
    h2 = mf.mf_prefix_hashes(other, 64)
    assert (h2[:3] == h[:3]).all() and (h2[3:] != h[3:]).all()
    # a longer sequence with the same prefix: the full blocks keep their hashes
    longer = np.concatenate([toks[:320], rng.integers(0, 9, size=50).astype(np.int32)])
    h3 = mf.mf_prefix_hashes(longer, 64)
    assert (h3[:5] == h[:5]).all() and h3[5] != h[5]
    assert len(mf.mf_prefix_hashes(np.zeros(0, np.int32), 64)) == 0


def test_cache_bookkeeping_without_copies(mf):
    """Creating a cache only cuts the pool into slots; validation happens on the host."""
    pool_bytes = 10 * 8 * 64 * 64 * 2 + 100
    d = mf.CacheDesc(4096, pool_bytes, 8, 64, mf.MF_BF16)
    h = ctypes.c_void_p()
    assert mf._lib.mf_cache_create(ctypes.byref(d), ctypes.byref(h)) == mf.MF_OK
    o = np.zeros(6, dtype=np.int64)
    assert mf._lib.mf_cache_stats(h, o.ctypes.data_as(ctypes.c_void_p)) == mf.MF_OK
    assert o.tolist() == [0, 0, 10, 0, 0, 0]
    # a get of nothing cached hits nothing and launches no copy
    hs = np.array([1, 2, 3], dtype=np.uint64)
    hit = ctypes.c_int32(-1)
    rc = mf._lib.mf_cache_get(h, 0, hs.ctypes.data_as(ctypes.c_void_p), 3, ctypes.c_void_p(4096),
                              ctypes.c_void_p(4096), ctypes.c_void_p(4096), 10, ctypes.byref(hit), None)
    assert hit.value == 0 or rc == mf.MF_ERR_CUDA  # the row_ptr write needs a device
    mf._lib.mf_cache_destroy(h)
    for bad in [mf.CacheDesc(4100, pool_bytes, 8, 64, mf.MF_BF16),     # misaligned pool
                mf.CacheDesc(4096, 100, 8, 64, mf.MF_BF16),            # smaller than one block
                mf.CacheDesc(4096, pool_bytes, 8, 48, mf.MF_BF16),     # block size
                mf.CacheDesc(None, pool_bytes, 8, 64, mf.MF_BF16)]:
        assert mf._lib.mf_cache_create(ctypes.byref(bad), ctypes.byref(h)) == mf.MF_ERR_INVALID
