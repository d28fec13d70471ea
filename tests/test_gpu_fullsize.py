"""Full-size parity on the five workloads, in the launch configuration bench.py times.

The oracle runs on sampled query blocks (the exact device bytes of each sampled row are
copied to the host); properties that hold at any size (bitwise layout identities, status
word clean, every row's kept set valid) are checked on all rows.
"""
import numpy as np
import pytest
import torch

import cross_model_attention_mf_b200 as mf
import synth
from synth import device as sdev
from tests.gpu_common import (assert_O_close, check_rows, compare_rows, host_bsr, oracle_O_rows,
                              oracle_pool, run_compress)

pytestmark = pytest.mark.gpu


def _status_ok():
    rc, bits = mf.mf_get_status()
    assert rc == mf.MF_OK and bits == 0, (rc, bits)


def _spread(n, k):
    return sorted(set([0, 1, n - 1] + np.linspace(0, n - 1, k).astype(int).tolist()))


def _valid_sets(w, bsr):
    """Every row: ascending, unique, diagonal present, indices <= qb."""
    rp, ci, nnz = host_bsr(bsr)
    assert rp[0] == 0 and rp[-1] == nnz and (np.diff(rp) >= 1).all()
    r = 0
    for s in range(len(w.lens)):
        for qb in range(w.nqb[s]):
            k = ci[rp[r]:rp[r + 1]]
            assert (np.diff(k) > 0).all() and k[-1] == qb and k[0] >= 0
            r += 1
    return nnz


def test_ministral_pair_full():
    w = synth.ALL["ministral_pair"]
    pack = sdev.fill_maps(sdev.alloc_maps(w), w, 0)
    bsr = run_compress(w, pack)
    _status_ok()
    nnz = _valid_sets(w, bsr)
    rows = [(0, qb) for qb in range(w.nqb[0])]  # every row: the oracle is fast enough here
    orows, nb = check_rows(w, pack, bsr, rows)
    assert nb == 0
    W = sdev.w_weights(w)
    V = sdev.v_contiguous(w, 0)
    cu = pack.cu_seqlens
    O = mf.mf_map_retrieve([bsr], [0], W, V, cu, cu, sdev.qblock_base(w), w.lens[0], w.h_r,
                           w.h_kv, total_q=w.tokens)[0]
    _status_ok()
    Wl, Vh = W[0].cpu().numpy(), V.cpu()
    for qb in _spread(w.nqb[0], 8):
        want, (lo, hi) = oracle_O_rows(w, orows, 0, qb, Wl, Vh, 0)
        got = O[qb * w.B + lo:qb * w.B + hi].float().cpu().numpy()
        assert_O_close(got, want, "bf16", f"ministral qb={qb}")
    print(f"ministral_pair nnz={nnz} density={nnz / w.causal_blocks:.4f}")


# The long-context sweep: tau x heavy-column count under both map readings.  Points that share
# (reading, heavy) share one 68.7 GB map fill, so they are listed next to each other.
LONG_POINTS = [(tau, heavy, reading) for reading in (1, 3) for heavy in (8, 64)
               for tau in (0.8, 0.9, 0.95, 0.99)]
# query blocks whose kept sets are compared (row 0, the last row and rows around the middle),
# and the blocks whose O rows are compared, on a few rows of each block
LONG_ROWS = [0, 1, 2, 31, 64, 127, 128, 129, 191, 254, 255]
LONG_O_BLOCKS = [0, 1, 128, 254, 255]
LONG_O_ROWS = [(0, 4), (60, 68), (120, 128)]
# most rows whose kept set may differ from the oracle's on one sweep point (only rows in the
# near-tie band may differ at all); the expectation is 0
LONG_MAX_MISMATCHED = 1

_long_maps = {}


def _long_pack(w):
    key = (w.n_heavy, w.reading)
    if key not in _long_maps:
        _long_maps.clear()
        torch.cuda.empty_cache()
        _long_maps[key] = sdev.fill_maps(sdev.alloc_maps(w), w, 0)
    return _long_maps[key]


@pytest.mark.parametrize("tau,heavy,reading", LONG_POINTS,
                         ids=[f"tau{t}-heavy{h}-R{r}" for t, h, r in LONG_POINTS])
def test_long_context_full(tau, heavy, reading):
    w = synth.ALL["long_context"].with_(tau=tau, n_heavy=heavy, reading=reading)
    pack = _long_pack(w)
    bsr = run_compress(w, pack, capacity=w.causal_blocks)
    _status_ok()
    nnz = _valid_sets(w, bsr)
    rows = [(0, qb) for qb in LONG_ROWS]
    res = compare_rows(w, pack, bsr, rows)
    orows, flagged, mism = res["orows"], res["flagged"], res["mismatched"]
    print(f"long_context tau={tau} heavy={heavy} R{reading} nnz={nnz} "
          f"density={nnz / w.causal_blocks:.4f} near-tie rows {flagged}/{len(rows)} "
          f"differing rows {mism}/{len(rows)}")
    # reading 1 has no near-tie row at all; under reading 3 the close-masses condition flags
    # rows, but the GPU's masses are far closer to the oracle's than the band, so the kept
    # sets are expected to match there as well
    if reading == 1:
        assert flagged == 0
    assert mism <= LONG_MAX_MISMATCHED
    W = sdev.w_weights(w)
    V = sdev.v_contiguous(w, 0)
    cu = pack.cu_seqlens
    O = mf.mf_map_retrieve([bsr], [0], W, V, cu, cu, sdev.qblock_base(w), w.lens[0], w.h_r,
                           w.h_kv, total_q=w.tokens)[0]
    _status_ok()
    Wl, Vh = W[0].cpu().numpy(), V.cpu()
    with oracle_pool() as pool:
        jobs = [(qb, rr, pool.submit(oracle_O_rows, w, orows, 0, qb, Wl, Vh, 0, row_range=rr))
                for qb in LONG_O_BLOCKS for rr in LONG_O_ROWS]
        for qb, rr, f in jobs:
            want, (lo, hi) = f.result()
            got = O[qb * w.B + lo:qb * w.B + hi].float().cpu().numpy()
            assert_O_close(got, want, "bf16", f"long tau={tau} heavy={heavy} R{reading} qb={qb} rows {lo}-{hi}")
    del bsr, O
    if (tau, heavy, reading) == LONG_POINTS[-1] or tau == 0.99:
        _long_maps.clear()
    torch.cuda.empty_cache()


def test_qwen_pair_all_layers():
    """40 sender layers compressed one at a time (each layer's dense maps are generated into
    one reused buffer), then all 36 receiver layers retrieved in one call."""
    w = synth.ALL["qwen_pair"]
    lm = w.layer_map()
    pack = sdev.alloc_maps(w)
    cap = 2048
    bsrs = []
    for l in range(w.n_sender_layers):
        sdev.fill_maps(pack, w, l)
        bsrs.append(run_compress(w, pack, capacity=cap, with_mass=False))
        _status_ok()
    for b in bsrs:
        _valid_sets(w, b)
    W = sdev.w_weights(w)
    T = w.tokens
    V = torch.empty((w.n_receiver_layers, T, w.h_kv, w.d), dtype=torch.bfloat16, device="cuda")
    for l in range(w.n_receiver_layers):
        V[l] = sdev.v_contiguous(w, l)
    qbase = sdev.qblock_base(w)
    cu = pack.cu_seqlens
    O = mf.mf_map_retrieve(bsrs, lm, W, V, cu, cu, qbase, max(w.lens), w.h_r, w.h_kv, total_q=T,
                           v_layer_stride=V[0].numel())
    _status_ok()
    starts = np.concatenate([[0], np.cumsum(w.lens)])
    for l_r in (0, 17, 35):
        l_s = lm[l_r]
        sdev.fill_maps(pack, w, l_s)
        rows = [(s, qb) for s in range(len(w.lens)) for qb in (0, w.nqb[s] // 2, w.nqb[s] - 1)]
        orows, nb = check_rows(w, pack, bsrs[l_s], rows, values=True)
        assert nb == 0
        Wl, Vh = W[l_r].cpu().numpy(), V[l_r].cpu()
        for (s, qb) in rows:
            want, (lo, hi) = oracle_O_rows(w, orows, s, qb, Wl, Vh, 0, k_start=int(starts[s]))
            got = O[l_r, starts[s] + qb * w.B + lo:starts[s] + qb * w.B + hi].float().cpu().numpy()
            assert_O_close(got, want, "bf16", f"qwen l_r={l_r} s={s} qb={qb}")
    # the one-call batch equals single-layer calls
    O5 = mf.mf_map_retrieve(bsrs, lm, W, V, cu, cu, qbase, max(w.lens), w.h_r, w.h_kv,
                            total_q=T, l_r_range=(5, 6), v_layer_stride=V[0].numel())
    assert torch.equal(O5[0], O[5])
    del pack, bsrs, V, O
    torch.cuda.empty_cache()


def test_routing_batch_chunked_paged():
    """16 varlen sequences, chunked prefill (2048-token query chunks against the full prefix)
    over a shuffled paged V: chunk results equal the whole-sequence result bit for bit, and
    sampled rows match the oracle (which walks the same block table)."""
    w = synth.ALL["routing_batch"]
    pack = sdev.fill_maps(sdev.alloc_maps(w), w, 0)
    bsr = run_compress(w, pack, capacity=8192)
    _status_ok()
    _valid_sets(w, bsr)
    W = sdev.w_weights(w)
    V = sdev.v_contiguous(w, 0)
    Vp, table = sdev.v_paged(w, V)
    qbase = sdev.qblock_base(w)
    cu = pack.cu_seqlens
    whole = mf.mf_map_retrieve([bsr], [0], W, Vp, cu, cu, qbase, max(w.lens), w.h_r, w.h_kv,
                               total_q=w.tokens, paged=(table, w.page_size))[0]
    parts = [[] for _ in w.lens]
    for step in synth.chunks(w):
        cu_q, cu_k, mq = sdev.step_tensors(step)
        Oc = mf.mf_map_retrieve([bsr], [0], W, Vp, cu_q, cu_k, qbase, mq, w.h_r, w.h_kv,
                                total_q=int(cu_q[-1]), paged=(table, w.page_size))[0]
        q = cu_q.cpu().numpy()
        for s in range(len(w.lens)):
            if q[s + 1] > q[s]:
                parts[s].append(Oc[q[s]:q[s + 1]])
    _status_ok()
    chunked = torch.cat([torch.cat(p) for p in parts])
    assert torch.equal(chunked, whole)
    starts = np.concatenate([[0], np.cumsum(w.lens)])
    tab = table.cpu().numpy()
    Vph = Vp.cpu()
    Wl = W[0].cpu().numpy()
    rows = [(s, qb) for s in (0, 5, 11, 15) for qb in (0, w.nqb[s] // 2, w.nqb[s] - 1)]
    orows, nb = check_rows(w, pack, bsr, rows)
    assert nb == 0
    for (s, qb) in rows:
        want, (lo, hi) = oracle_O_rows(w, orows, s, qb, Wl, Vph, 0, block_table=tab[s],
                                       page_size=w.page_size)
        got = whole[starts[s] + qb * w.B + lo:starts[s] + qb * w.B + hi].float().cpu().numpy()
        assert_O_close(got, want, "bf16", f"routing s={s} qb={qb}")
    del pack, bsr, Vp, whole
    torch.cuda.empty_cache()
