"""The seeded input recipe (CPU side): invariants of the generated maps, V, W and layouts."""
import numpy as np
import pytest
import torch

import synth
from synth import maps as smaps
from synth import rng


def test_splitmix64_reference_values():
    # SplitMix64 seeded with 0: the first outputs of the published generator
    x = rng.draw(np.uint64(0), np.arange(3, dtype=np.uint64))
    assert [int(v) for v in x] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_normals_are_standard():
    z = rng.normal(rng.stream_key(0, rng.TAG_V), np.arange(200000, dtype=np.uint64))
    assert abs(float(z.mean())) < 0.01
    assert abs(float(z.std()) - 1.0) < 0.01
    assert np.isfinite(z).all()


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("reading", [1, 3])
def test_maps_are_causal_row_softmax(dt, reading):
    L, B, h_s = 77, 16, 3
    A = smaps.gen_maps(L, B, h_s, 5, seed=2, reading=reading, dtype=dt).float().numpy().astype(np.float64)
    Lp = A.shape[1]
    assert Lp == 80
    i = np.arange(Lp)[:, None]
    j = np.arange(Lp)[None, :]
    causal = (j <= i) & (i < L)
    assert (A[:, ~causal] == 0).all()
    assert (A[:, causal] >= 0).all()
    sums = A[:, :L, :].sum(axis=2)
    # round-to-nearest into bf16 (8 significant bits) moves each entry by at most 2**-8 of itself
    tol = 1e-6 if dt == "f32" else 2.0 ** -8 + 1e-6
    assert np.abs(sums - 1.0).max() <= tol


def test_maps_follow_recipe_terms():
    """Sinks and heavy columns receive more mass than the local decay alone would give."""
    L, B, h_s = 512, 64, 2
    A = smaps.gen_maps(L, B, h_s, 8, seed=1, reading=3, dtype="f32").numpy()
    hv = smaps.heavy_columns(1, 0, 0, 0, L, 8)
    far = A[0, 400:512]
    plain = np.setdiff1d(np.arange(0, 300), np.concatenate([hv, np.arange(4)]))
    assert far[:, :4].mean() > 5 * far[:, plain].mean()
    hv_far = hv[hv < 300]
    if len(hv_far):
        assert far[:, hv_far].mean() > 2 * far[:, plain].mean()


def test_heavy_columns_distinct_and_seeded():
    a = smaps.heavy_columns(0, 1, 2, 3, 1000, 64)
    b = smaps.heavy_columns(0, 1, 2, 3, 1000, 64)
    c = smaps.heavy_columns(1, 1, 2, 3, 1000, 64)
    assert len(set(a.tolist())) == 64 and a.min() >= 0 and a.max() < 1000
    assert (a == b).all() and not (a == c).all()
    assert sorted(smaps.heavy_columns(0, 0, 0, 0, 5, 5).tolist()) == [0, 1, 2, 3, 4]
    assert sorted(smaps.heavy_columns(0, 0, 0, 0, 3, 16).tolist()) == [0, 1, 2]


def test_v_and_w_distributions():
    W = smaps.gen_w(3, 32, 32, seed=0).numpy()
    assert W.shape == (3, 32, 32) and W.dtype == np.float32
    assert abs(W.var() - 1.0 / 32) < 0.1 / 32
    V = smaps.gen_v(4096, 2, 16, seed=0, dtype="bf16")
    assert V.dtype == torch.bfloat16 and abs(float(V.float().std()) - 1) < 0.02


def test_workloads_shapes():
    w = synth.ALL["qwen_pair"]
    lm = w.layer_map()
    assert lm == [(78 * l + 35) // 70 for l in range(36)]
    assert sorted(set(range(40)) - set(lm)) == [5, 15, 24, 34]
    assert sum(w.nqb) == 256 and w.tokens == 16384
    c5 = synth.ALL["routing_batch"]
    assert len(c5.lens) == 16 and all(1024 <= L <= 8192 for L in c5.lens)
    assert synth.ALL["long_context"].causal_blocks == 256 * 257 // 2


def test_chunks_cover_every_query_once():
    w = synth.ALL["routing_batch"]
    seen = [0] * len(w.lens)
    for step in synth.chunks(w):
        for s, (q, k) in enumerate(step):
            if q:
                assert k - q == seen[s] and (k - q) % w.B == 0
                seen[s] = k
    assert seen == list(w.lens)


def test_page_table_is_a_permutation():
    w = synth.ALL["routing_batch"]
    table, total = synth.page_table(w)
    used = table[table >= 0]
    assert total == sum(-(-L // w.page_size) for L in w.lens)
    assert sorted(used.tolist()) == list(range(total))
    assert (np.diff(used) != 1).any()  # shuffled


def test_qk_recipe_is_seeded_and_structured():
    """synth.qk: same seed, same bytes; another seed, other bytes; the causal attention it
    induces is concentrated (a recency peak, with sinks and heavy keys taking the rest), the
    structure that makes block selection keep few blocks."""
    import math

    import numpy as np
    import torch

    import oracle
    from synth.qk import gen_qk
    Q, K = gen_qk((1000,), 4, 2, 128, 8, seed=0)
    Q2, K2 = gen_qk((1000,), 4, 2, 128, 8, seed=0)
    Q3, _ = gen_qk((1000,), 4, 2, 128, 8, seed=1)
    assert Q.dtype == torch.bfloat16 and Q.shape == (1000, 4, 128) and K.shape == (1000, 2, 128)
    assert torch.equal(Q, Q2) and torch.equal(K, K2) and not torch.equal(Q, Q3)
    A = oracle.qk_maps(Q, K, 1000, 64, 1.0 / math.sqrt(128))
    for i in (299, 600, 999):
        row = A[0, i, :i + 1]
        assert np.sort(row)[::-1][:10].sum() > 0.9      # ten keys hold most of the mass
        assert row[i - 7:i + 1].sum() > 0.5             # the recency peak
