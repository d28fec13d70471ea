"""Host logic of bench.py's end-to-end leg: the copy plan for the dense maps (no GPU)."""
from types import SimpleNamespace

import numpy as np
import pytest

import bench
import synth
from synth import device as sdev


@pytest.mark.parametrize("name", ["tiny", "ministral_pair", "qwen_pair", "routing_batch"])
@pytest.mark.parametrize("group", [1, 3, 8])
def test_causal_slabs_cover_every_causal_block(name, group):
    """Every key block j <= i of every query row i of every head and sequence lies in some
    slab, and no slab leaves its sequence's [h][Lp][Lp] maps."""
    w = synth.ALL[name]
    offs, total = sdev.map_offsets(w)
    pack = SimpleNamespace(offsets=offs)
    slabs = bench.causal_slabs(w, pack, group)
    B = w.B
    for s, L in enumerate(w.lens):
        Lp = -(-L // B) * B
        nqb = -(-L // B)
        base = offs[s]
        # covered[h, qb] = number of key columns copied for query block qb of head h
        covered = np.zeros((w.h_s, nqb), dtype=np.int64)
        for off, rows, width, pitch in slabs:
            rel = off - base
            if rel < 0 or rel >= w.h_s * Lp * Lp:
                continue
            assert pitch == Lp and width <= Lp
            h, r0 = divmod(rel, Lp * Lp)
            i0, c0 = divmod(r0, Lp)
            assert c0 == 0 and i0 % B == 0
            assert i0 + rows <= L  # rows past the sequence are never copied
            for qb in range(i0 // B, -(-(i0 + rows) // B)):
                covered[h, qb] = max(covered[h, qb], width)
        need = np.array([(qb + 1) * B for qb in range(nqb)])
        assert (covered >= need[None, :]).all()
        assert total >= base + w.h_s * Lp * Lp


def test_oracle_config_sample_on_the_host():
    """The bench's per-config CPU leg on the tiny workload with maps built by the CPU recipe:
    the reported tokens, core count and near-tie count are consistent."""
    import torch
    from synth import maps as sm
    w = synth.ALL["tiny"]
    pack = sdev.fill_maps(sdev.alloc_maps(w, "cpu"), w, 0, use_gpu=False)
    W = np.asarray(sm.gen_w(1, w.h_r, w.h_s, seed=w.seed))[0]
    V = torch.as_tensor(sm.gen_v(w.lens[0], w.h_kv, w.d, seed=w.seed))
    out = bench.oracle_config_sample(w, pack, W, V, n_rows=4)
    assert out["kind"] == "oracle" and out["cores"] >= 1
    assert out["near_tie_rows"] == 0  # the tiny workload has no near-tie row
    assert out["value"] > 0 and out["seconds"] > 0
    assert "4 of 8 query blocks" in out["sample"]
