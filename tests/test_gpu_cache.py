"""Prefix-hash block cache on the GPU: a request that shares a prefix with a cached one gets,
bit for bit, the cached rows of that prefix; retrieval over the assembled BSR equals retrieval
over the original rows; eviction follows least-recent use; assembly on a side stream overlaps
work on the main stream and is ordered by an event (MapFlow page "MapFlow开源:大模型换班,Prefill
为何能快20%?", section "存不下、读得慢?三个工程优化手段", subsection 2)."""
import numpy as np
import pytest
import torch

import cross_model_attention_mf_b200 as mf
import synth
from synth import device as sdev
from tests.gpu_common import run_compress

pytestmark = pytest.mark.gpu


def _status_ok():
    rc, bits = mf.mf_get_status()
    assert rc == mf.MF_OK and bits == 0, (rc, bits)


def _request(L, seed=0):
    w = synth.Workload("cache", (L,), B=64, h_s=32, h_r=32, h_kv=8, d=128, dtype="bf16",
                       tau=0.95, n_heavy=16, reading=3, seed=seed)
    pack = sdev.fill_maps(sdev.alloc_maps(w), w, 0)
    return w, pack, run_compress(w, pack)


def _pool(blocks, h_s=32, B=64):
    return torch.empty(blocks * h_s * B * B * 2, dtype=torch.uint8, device="cuda")


def test_shared_prefix_gets_cached_rows_bitwise():
    w, pack, bsr = _request(700)
    rng = np.random.default_rng(1)
    toks = rng.integers(0, 50000, size=700).astype(np.int32)
    cache = mf.BlockCache(_pool(400), 32, 64)
    hA = mf.mf_prefix_hashes(toks, 64)
    assert cache.put(0, bsr, hA) == len(hA)
    # request B: the same first 5 blocks (320 tokens), then other tokens
    toksB = np.concatenate([toks[:320], rng.integers(0, 50000, size=200).astype(np.int32)])
    hB = mf.mf_prefix_hashes(toksB, 64)
    out = mf.alloc_bsr(len(hB), 200, 32, 64, torch.bfloat16, "cuda")
    hit = cache.get(0, hB, out)
    torch.cuda.synchronize()
    assert hit == 5
    rp = bsr.row_ptr.cpu().numpy()
    n = rp[5]
    assert out.row_ptr[:6].cpu().tolist() == rp[:6].tolist()
    assert torch.equal(out.col_idx[:n], bsr.col_idx[:n])
    assert torch.equal(out.values[:n], bsr.values[:n])
    # retrieval over the assembled rows equals retrieval over the original rows
    W = sdev.w_weights(w)
    V = sdev.v_contiguous(w, 0)
    qb = torch.zeros(1, dtype=torch.int32, device="cuda")
    cu_a = torch.tensor([0, 700], dtype=torch.int32, device="cuda")
    cu_b = torch.tensor([0, 320], dtype=torch.int32, device="cuda")
    O_a = mf.mf_map_retrieve([bsr], [0], W, V, cu_a, cu_a, qb, 700, 32, 8, total_q=700)[0]
    O_b = mf.mf_map_retrieve([out], [0], W, V[:320].contiguous(), cu_b, cu_b, qb, 320, 32, 8,
                             total_q=320)[0]
    assert torch.equal(O_b, O_a[:320])
    st = cache.stats()
    assert st["rows"] == 11 and st["hits"] == 5 and st["misses"] == 1 and st["evicted"] == 0
    _status_ok()


def test_layers_are_separate_and_eviction_is_lru():
    w, pack, bsr = _request(640)
    rp = bsr.row_ptr.cpu().numpy()
    sizes = np.diff(rp)
    toks = np.arange(640, dtype=np.int32)
    h = mf.mf_prefix_hashes(toks, 64)
    need = int(sizes[:4].sum())
    cache = mf.BlockCache(_pool(need), 32, 64)     # room for rows 0-3 only
    assert cache.put(0, bsr, h[:4], row0=0, nrows=4) == 4
    out = mf.alloc_bsr(10, 64, 32, 64, torch.bfloat16, "cuda")
    assert cache.get(1, h, out) == 0               # another layer: nothing
    assert cache.get(0, h[:2], out) == 2           # rows 0, 1 become the most recent
    # row 4 needs room: the least recently used rows (3, then 2) go first
    assert cache.put(0, bsr, h[4:5], row0=4, nrows=1) == 1
    st = cache.stats()
    assert st["evicted"] >= 1 and st["rows"] == 5 - st["evicted"]
    hit = cache.get(0, h, out)
    assert hit == 2                                # rows 0, 1 survive; the prefix breaks at 2
    torch.cuda.synchronize()
    n = rp[2]
    assert torch.equal(out.values[:n], bsr.values[:n])
    _status_ok()


def test_assembly_on_a_side_stream_is_ordered_by_an_event():
    w, pack, bsr = _request(1000, seed=3)
    toks = np.arange(1000, dtype=np.int32) * 7
    h = mf.mf_prefix_hashes(toks, 64)
    cache = mf.BlockCache(_pool(600), 32, 64)
    cache.put(0, bsr, h)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    out = mf.alloc_bsr(len(h), 600, 32, 64, torch.bfloat16, "cuda")
    out.values.zero_()
    torch.cuda.synchronize()
    a = torch.randn(4096, 4096, device="cuda", dtype=torch.bfloat16)
    busy = a @ a  # the receiver's own first layers stand here  # noqa: F841
    with torch.cuda.stream(side):
        hit = cache.get(0, h, out, stream=side)
        ev = torch.cuda.Event()
        ev.record(side)
    torch.cuda.current_stream().wait_event(ev)
    n = int(bsr.row_ptr[-1].item())
    assert hit == len(h)
    assert torch.equal(out.values[:n], bsr.values[:n])
    assert torch.equal(out.row_ptr, bsr.row_ptr)
    _status_ok()


def test_one_put_larger_than_the_pool_keeps_the_latest_rows_intact():
    """Rows evicted inside one put must not leave their data in the slots of later rows."""
    w, pack, bsr = _request(900, seed=5)
    rp = bsr.row_ptr.cpu().numpy()
    sizes = np.diff(rp)
    h = mf.mf_prefix_hashes(np.arange(900, dtype=np.int32) + 11, 64)
    cap = int(sizes[-3:].sum())                    # room for about the last three rows
    cache = mf.BlockCache(_pool(cap), 32, 64)
    cache.put(0, bsr, h)
    st = cache.stats()
    assert st["evicted"] > 0 and st["used"] <= cap
    out = mf.alloc_bsr(1, 64, 32, 64, torch.bfloat16, "cuda")
    last = len(h) - 1
    assert cache.get(0, h[last:], out) == 1
    torch.cuda.synchronize()
    n0, n1 = rp[last], rp[last + 1]
    assert torch.equal(out.values[:n1 - n0], bsr.values[n0:n1])
    assert torch.equal(out.col_idx[:n1 - n0], bsr.col_idx[n0:n1])
    _status_ok()


def test_put_from_an_overflowed_bsr_caches_no_short_row():
    """A compression that ran out of capacity wrote only the first capacity_blocks blocks; the
    rows that reach past that point are incomplete and must not be cached (a later hit would
    return a short row with no error)."""
    w, pack, full = _request(700)
    rp = full.row_ptr.cpu().numpy()
    cap = int(rp[6]) - 1  # rows 0-4 fit; row 5 loses its last block
    bsr = run_compress(w, pack, capacity=cap)
    rc, bits = mf.mf_get_status()
    assert rc == mf.MF_ERR_CAPACITY and bits == 2, (rc, bits)
    assert bsr.row_ptr.cpu().tolist() == rp.tolist()  # row_ptr holds the true counts
    toks = np.random.default_rng(3).integers(0, 50000, size=700).astype(np.int32)
    h = mf.mf_prefix_hashes(toks, 64)
    cache = mf.BlockCache(_pool(400), 32, 64)
    assert cache.put(0, bsr, h) == 5
    out = mf.alloc_bsr(len(h), 400, 32, 64, torch.bfloat16, "cuda")
    assert cache.get(0, h, out) == 5
    torch.cuda.synchronize()
    n = int(rp[5])
    assert out.row_ptr[:6].cpu().tolist() == rp[:6].tolist()
    assert torch.equal(out.values[:n], full.values[:n])
    # the complete rows, put from the full BSR, then fill the rest of the request
    assert cache.put(0, full, h) == len(h) - 5
    assert cache.get(0, h, out) == len(h)
    torch.cuda.synchronize()
    assert torch.equal(out.values[:int(rp[-1])], full.values[:int(rp[-1])])
    _status_ok()


def test_matches_the_host_model():
    """A sequence of puts and gets over two layers and three requests (two sharing a prefix),
    in a pool small enough to evict: after every operation the library's return value, its
    counters and every assembled row (row_ptr, col_idx, values, bit for bit) equal those of
    the plain host model of the cache (oracle/cache_model.py)."""
    import oracle
    from oracle.cache_model import PrefixCacheModel, prefix_hashes

    rng = np.random.default_rng(7)
    toks_a = rng.integers(0, 50000, size=700).astype(np.int32)
    toks_b = np.concatenate([toks_a[:320], rng.integers(0, 50000, size=380).astype(np.int32)])
    toks_c = rng.integers(0, 50000, size=700).astype(np.int32)
    hashes = {}
    for name, toks in (("A", toks_a), ("B", toks_b), ("C", toks_c)):
        h = mf.mf_prefix_hashes(toks, 64)
        assert h.tolist() == prefix_hashes(toks, 64)
        hashes[name] = h
    # compressed layers: layer 0 from request A's maps (its rows serve every request in this
    # test: only the keys differ), layer 1 from another map layer
    w, pack, bsr0 = _request(700)
    sdev.fill_maps(pack, w, 1)
    bsr1 = run_compress(w, pack)
    _status_ok()
    src = {}
    for layer, b in ((0, bsr0), (1, bsr1)):
        raw, _ = oracle.as_raw(b.values[:int(b.nnz.cpu()[0])].cpu())
        src[layer] = (b, b.row_ptr.cpu().numpy(), b.col_idx.cpu().numpy(), raw)
    n_slots = 60
    cache = mf.BlockCache(_pool(n_slots), 32, 64)
    model = PrefixCacheModel(n_slots)
    out = mf.alloc_bsr(11, 200, 32, 64, torch.bfloat16, "cuda")

    def put(layer, req, row0, n):
        b, rp, ci, raw = src[layer]
        h = hashes[req][row0:row0 + n]
        got = cache.put(layer, b, h, row0=row0, nrows=n)
        want = model.put(layer, rp, ci, raw, b.capacity, row0, h.tolist())
        assert got == want, ("put", layer, req, row0, n, got, want)

    def get(layer, req, capacity=200):
        out.row_ptr.fill_(-1)
        o = mf.BSR(out.row_ptr, out.col_idx, out.values[:capacity], out.nnz)
        got = cache.get(layer, hashes[req], o)
        want, rp, ci, vals = model.get(layer, hashes[req].tolist(), capacity)
        assert got == want, ("get", layer, req, got, want)
        torch.cuda.synchronize()
        assert out.row_ptr[:got + 1].cpu().tolist() == rp
        n = rp[-1]
        assert out.col_idx[:n].cpu().tolist() == ci
        if n:
            raw, _ = oracle.as_raw(out.values[:n].cpu())
            assert raw.tobytes() == vals.tobytes()

    ops = [("put", 0, "A", 0, 11), ("get", 0, "B"), ("put", 1, "A", 0, 6), ("put", 0, "C", 0, 11),
           ("get", 0, "A"), ("get", 1, "B"), ("put", 0, "B", 0, 11), ("get", 0, "C"),
           ("get", 0, "A", 30), ("put", 1, "C", 3, 8), ("get", 1, "A"), ("get", 0, "B"),
           ("put", 0, "A", 5, 6), ("get", 0, "A")]
    for op in ops:
        if op[0] == "put":
            put(*op[1:])
        else:
            get(*op[1:])
        st = cache.stats()
        ms = model.stats()
        assert st == ms, (op, st, ms)
    assert cache.stats()["evicted"] > 0
    _status_ok()
