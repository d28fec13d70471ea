"""Pins of the CPU oracle to facts outside itself (no GPU).

Each oracle function is checked against something it does not share code with:
  - block statistics: brute-force Python loops and numpy masked sums;
  - selection: exhaustive subset search in exact rational arithmetic (the fewest
    blocks reaching tau), the greedy exchange property, hand-checked ties;
  - kept-block write: numpy slicing with a causal mask, byte for byte;
  - retrieval: the dense receiver map (sum_s W A_s) times V in numpy at tau = 1,
    textbook causal softmax attention (numpy and torch SDPA) with W = I and maps
    built from Q, K, one-hot W rows, GQA by repeating KV heads, linearity, and
    the layout identities (chunked = whole, paged = contiguous);
  - a worked example whose numbers are derived by hand in the comments.
A plausible slip in the oracle (dropped term, wrong sign or index, transposed
operand, off-by-one in a mask or a block edge) breaks at least one of these.
"""
import itertools
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import maps as smaps

RNG = np.random.default_rng(12345)


def causal_mask(L, Lp):
    i = np.arange(Lp)[:, None]
    j = np.arange(Lp)[None, :]
    return (j <= i) & (i < L) & (j < L)


def dense_maps(h_s, L, B, rng=RNG, garbage=True):
    """Random non-negative maps [h_s, Lp, Lp] float32 with garbage outside the causal part
    (the oracle must ignore it)."""
    Lp = -(-L // B) * B
    a = rng.random((h_s, Lp, Lp)).astype(np.float32)
    if garbage:
        a = np.where(causal_mask(L, Lp)[None], a, np.float32(7.0))
    return a


# ----------------------------------------------------------------------- worked example

def test_worked_example_by_hand():
    """h_s = 2, L = 5, B = 2 (Lp = 6, three query blocks, ragged last block).
    Sender maps (causal part; 9.0 marks entries the method must ignore):
        A_0 row i, col j = 1 for j <= i          (all ones)
        A_1 row i, col j = (j + 1) / 8 for j <= i
    Block masses, head-summed, counting only j <= i < 5:
      qb 0 (rows 0,1): kb0 = A_0: 3 entries -> 3 ; A_1: (1 + 1 + 2)/8 = 0.5  -> 3.5
      qb 1 (rows 2,3): kb0: A_0 4 -> 4 ; A_1 rows 2,3 cols 0,1: 2*(1+2)/8 = 0.75 -> 4.75
                       kb1: A_0 cols 2,3: row2 {2}, row3 {2,3} -> 3 ; A_1: (3 + 3 + 4)/8 = 1.25 -> 4.25
      qb 2 (row 4 only): kb0: 2 + (1+2)/8 = 2.375 ; kb1: 2 + (3+4)/8 = 2.875 ;
                         kb2: col 4 only -> 1 + 5/8 = 1.625
    Selection, tau = 0.5:
      qb 2: total 6.875, target 3.4375; diagonal 1.625 < target; next kb1 (2.875):
            4.5 >= target -> kept {1, 2}.
      qb 1: total 9.0, target 4.5; diagonal 4.25 < 4.5; add kb0 -> kept {0, 1}.
      qb 0: kept {0}.
    Retrieval with h_r = 1, W = [1, -1], h_kv = 1, d = 1, V[j] = j + 1 (j < 5):
      row 4 (qb 2, kept kb1 and kb2; kb0 is dropped):
        P[j] = A_0[4,j] - A_1[4,j] = 1 - (j+1)/8 for j in {2, 3, 4} -> 5/8, 4/8, 3/8
        O = 5/8 * 3 + 4/8 * 4 + 3/8 * 5 = (15 + 16 + 15) / 8 = 46/8 = 5.75
      row 2 (qb 1, kept {0, 1}): P[j] = 1 - (j+1)/8 for j <= 2 -> 7/8, 6/8, 5/8
        O = 7/8 * 1 + 6/8 * 2 + 5/8 * 3 = (7 + 12 + 15) / 8 = 34/8 = 4.25
    """
    L, B, Lp = 5, 2, 6
    A = np.full((2, Lp, Lp), 9.0, dtype=np.float32)
    for i in range(L):
        for j in range(i + 1):
            A[0, i, j] = 1.0
            A[1, i, j] = (j + 1) / 8.0
    res = oracle.compress_seq(A, L, B, 0.5)
    np.testing.assert_array_equal(res["masses"][0], [3.5])
    np.testing.assert_array_equal(res["masses"][1], [4.75, 4.25])
    np.testing.assert_array_equal(res["masses"][2], [2.375, 2.875, 1.625])
    assert res["kept"][0].tolist() == [0]
    assert res["kept"][1].tolist() == [0, 1]
    assert res["kept"][2].tolist() == [1, 2]
    W = np.array([[1.0, -1.0]], dtype=np.float32)
    V = (np.arange(L, dtype=np.float32) + 1.0).reshape(L, 1, 1)
    O4 = oracle.retrieve_block(res["values"][2], res["kept"][2], 2, B, W, V, 1, (0, 1))
    assert O4[0, 0, 0] == pytest.approx(5.75, abs=1e-15)
    O2 = oracle.retrieve_block(res["values"][1], res["kept"][1], 1, B, W, V, 1, (0, 1))
    assert O2[0, 0, 0] == pytest.approx(4.25, abs=1e-15)


# ----------------------------------------------------------------------- block statistics

@pytest.mark.parametrize("L,B,h_s", [(7, 4, 2), (16, 4, 3), (13, 8, 2), (1, 4, 1)])
def test_masses_brute_force(L, B, h_s):
    A = dense_maps(h_s, L, B)
    nqb = -(-L // B)
    for qb in range(nqb):
        got = oracle.row_masses(A[:, qb * B:(qb + 1) * B, :], L, B, qb)
        for kb in range(qb + 1):
            want = 0.0
            for s in range(h_s):
                for i in range(qb * B, min((qb + 1) * B, L)):
                    for j in range(kb * B, min((kb + 1) * B, L)):
                        if j <= i:
                            want += float(A[s, i, j])
            assert got[kb] == pytest.approx(want, rel=1e-13, abs=0)


def test_masses_numpy_blocks_bf16():
    L, B, h_s = 45, 8, 3
    A = torch.from_numpy(dense_maps(h_s, L, B)).to(torch.bfloat16)
    Af = A.float().numpy().astype(np.float64)
    Lp = Af.shape[1]
    Am = np.where(causal_mask(L, Lp)[None], Af, 0.0)
    for qb in range(-(-L // B)):
        got = oracle.row_masses(A[:, qb * B:(qb + 1) * B, :], L, B, qb)
        want = Am[:, qb * B:(qb + 1) * B, :(qb + 1) * B].reshape(h_s, B, qb + 1, B).sum(axis=(0, 1, 3))
        np.testing.assert_allclose(got, want, rtol=1e-13, atol=0)


def test_masses_constant_closed_form():
    """Constant c on the causal part: an interior block holds B*B causal entries, a diagonal
    block B*(B+1)/2, and the ragged last row block of L = qb*B + t rows holds t*B (interior)
    or t*(t+1)/2 (diagonal)."""
    L, B, h_s, c = 27, 8, 3, 0.25
    Lp = 32
    A = np.broadcast_to(np.where(causal_mask(L, Lp), c, 5.0), (h_s, Lp, Lp)).astype(np.float32).copy()
    for qb in range(4):
        m = oracle.row_masses(A[:, qb * B:(qb + 1) * B, :], L, B, qb)
        t = min(B, L - qb * B)
        for kb in range(qb + 1):
            if kb < qb:
                want = h_s * c * t * B
            else:
                want = h_s * c * t * (t + 1) / 2
            assert m[kb] == want


# ----------------------------------------------------------------------- selection

def _brute_min_sets(mass, qb, tau):
    """All minimum-cardinality subsets containing the diagonal whose exact mass reaches
    tau * total."""
    fm = [Fraction(float(x)) for x in mass]
    total = sum(fm)
    target = Fraction(tau) * total
    others = [k for k in range(qb)]
    for size in range(0, qb + 1):
        hits = []
        for comb in itertools.combinations(others, size):
            if fm[qb] + sum(fm[k] for k in comb) >= target:
                hits.append(tuple(sorted(comb + (qb,))))
        if hits:
            return hits, fm
    raise AssertionError("no subset reaches tau")


@pytest.mark.parametrize("trial", range(60))
def test_selection_brute_force(trial):
    rng = np.random.default_rng(1000 + trial)
    qb = int(rng.integers(0, 10))
    # dyadic masses with deliberate ties, dyadic tau: every sum is exact in float64
    mass = rng.integers(0, 6, size=qb + 1).astype(np.float64) / 64.0
    if mass.sum() == 0:
        mass[qb] = 1.0 / 64
    tau = float(rng.choice([0.25, 0.5, 0.625, 0.75, 0.875, 0.9375, 1.0]))
    kept, info = oracle.select(mass, qb, tau)
    hits, fm = _brute_min_sets(mass, qb, tau)
    assert tuple(kept.tolist()) in hits, (mass, tau, kept, hits)
    # greedy exchange property: no minimum set carries more mass
    assert sum(fm[k] for k in kept) == max(sum(fm[k] for k in h) for h in hits)
    # tie rule: among maximum-mass minimum sets, the walk prefers smaller key-block indices
    best = max(sum(fm[k] for k in h) for h in hits)
    cands = sorted(h for h in hits if sum(fm[k] for k in h) == best)
    key = lambda h: sorted(((-fm[k], k) for k in h if k != qb))
    assert tuple(kept.tolist()) == min(cands, key=key)
    assert kept.tolist() == sorted(kept.tolist()) and qb in kept.tolist()


def test_selection_ties_and_edges():
    # four equal blocks, half the mass: the diagonal plus the lowest index
    assert oracle.select(np.ones(4), 3, 0.5)[0].tolist() == [0, 3]
    # tau <= 0 keeps only the diagonal; one block row keeps itself
    assert oracle.select(np.array([5.0, 1.0, 0.0]), 2, 0.0)[0].tolist() == [2]
    assert oracle.select(np.array([0.0]), 0, 0.95)[0].tolist() == [0]
    # tau = 1 keeps every block that adds mass and drops exact zeros
    assert oracle.select(np.array([1.0, 0.0, 2.0, 0.0, 1.0]), 4, 1.0)[0].tolist() == [0, 2, 4]
    # masses ranked by size, not by index
    assert oracle.select(np.array([0.1, 0.6, 0.2, 0.1]), 3, 0.7)[0].tolist() == [1, 3]


def test_selection_invariants_generated_maps():
    w = synth.ALL["tiny"]
    L, B = w.lens[0], w.B
    A = smaps.gen_maps(L, B, w.h_s, w.n_heavy, seed=3, dtype="f32")
    perm = [2, 0, 3, 1]
    Ap = A[perm].contiguous()
    prev = None
    for tau in (0.5, 0.8, 0.9, 0.95, 0.99, 1.0):
        r = oracle.compress_seq(A, L, B, tau)
        rp = oracle.compress_seq(Ap, L, B, tau)
        counts = []
        for qb, kept in r["kept"].items():
            m = r["masses"][qb]
            total = m.sum()
            km = m[kept].sum()
            assert km >= tau * total * (1 - 1e-12)
            # minimality: without the last block the walk added, the target is missed
            if len(kept) > 1:
                others = sorted((x for x in kept if x != qb), key=lambda k: (-m[k], k))
                assert km - m[others[-1]] < tau * total
            if not oracle.is_boundary(r["info"][qb], tau):
                assert rp["kept"][qb].tolist() == kept.tolist()  # sender-head order is irrelevant
            counts.append(len(kept))
        if prev is not None:
            assert all(a >= b for a, b in zip(counts, prev))  # monotone in tau
        prev = counts


# ----------------------------------------------------------------------- kept-block write

@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_gather_equals_masked_slices(dt):
    L, B, h_s = 21, 8, 2
    A = torch.from_numpy(dense_maps(h_s, L, B))
    if dt == "bf16":
        A = A.to(torch.bfloat16)
    raw, _ = oracle.as_raw(A)
    Lp = raw.shape[1]
    mask = causal_mask(L, Lp)
    for qb in range(-(-L // B)):
        for kb in range(qb + 1):
            got = oracle.gather_block(raw[:, qb * B:(qb + 1) * B, :], L, B, qb, kb)
            sl = (slice(None), slice(qb * B, (qb + 1) * B), slice(kb * B, (kb + 1) * B))
            want = np.where(mask[sl[1:]][None], raw[sl], 0).astype(raw.dtype)
            assert got.tobytes() == want.tobytes()


# ----------------------------------------------------------------------- retrieval

def _bsr_of(res):
    return lambda row: (res["kept"][row], res["values"][row])


def _dense_reference(A, L, W, V, h_kv):
    """(sum_s W[r,s] A_s) V_{g(r)} on the whole causal map, numpy float64, with GQA done
    the usual way: repeat each KV head h_r/h_kv times."""
    Af = A.float().numpy().astype(np.float64) if isinstance(A, torch.Tensor) else A.astype(np.float64)
    Lp = Af.shape[1]
    Am = np.where(causal_mask(L, Lp)[None], Af, 0.0)[:, :L, :L]
    P = np.einsum("rs,sij->rij", W.astype(np.float64), Am)
    h_r = W.shape[0]
    Vf = V.float().numpy().astype(np.float64) if isinstance(V, torch.Tensor) else V.astype(np.float64)
    Vrep = np.repeat(Vf, h_r // h_kv, axis=1)  # [L, h_r, d]
    return np.einsum("rij,jrd->ird", P, Vrep)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_tau_one_equals_dense(dt):
    L, B, h_s, h_r, h_kv, d = 37, 8, 3, 4, 2, 5
    A = smaps.gen_maps(L, B, h_s, 4, seed=7, dtype=dt)
    W = smaps.gen_w(1, h_r, h_s, seed=7)[0].numpy()
    V = smaps.gen_v(L, h_kv, d, seed=7, dtype=dt)
    res = oracle.compress_seq(A, L, B, 1.0)
    O = oracle.retrieve_step(_bsr_of(res), B, W, V, h_kv, [(L, L)], [0])
    want = _dense_reference(A, L, W, V, h_kv)
    np.testing.assert_allclose(O, want, rtol=1e-9, atol=1e-12)


def test_sparse_equals_dense_on_kept_blocks():
    """tau < 1: the oracle equals the dense product with the dropped blocks zeroed (numpy)."""
    L, B, h_s, h_r, h_kv, d = 64, 8, 4, 4, 1, 6
    A = smaps.gen_maps(L, B, h_s, 3, seed=11, dtype="f32")
    W = smaps.gen_w(1, h_r, h_s, seed=11)[0].numpy()
    V = smaps.gen_v(L, h_kv, d, seed=11)
    res = oracle.compress_seq(A, L, B, 0.8)
    keep = np.zeros((L, L), dtype=bool)
    for qb, kept in res["kept"].items():
        for kb in kept:
            keep[qb * B:(qb + 1) * B, kb * B:(kb + 1) * B] = True
    assert not keep.all()
    Ak = np.where(keep[None], A.numpy(), 0.0)
    O = oracle.retrieve_step(_bsr_of(res), B, W, V, h_kv, [(L, L)], [0])
    np.testing.assert_allclose(O, _dense_reference(Ak, L, W, V, h_kv), rtol=1e-9, atol=1e-12)


def test_identity_W_is_causal_attention():
    """Maps built as causal softmax(Q K^T / sqrt(dk)) per head, W = I, h_r = h_s = h_kv:
    the retrieved O is standard causal attention (numpy and torch SDPA, float64)."""
    L, B, H, dk, d = 40, 8, 3, 16, 8
    rng = np.random.default_rng(5)
    Q = rng.standard_normal((H, L, dk))
    K = rng.standard_normal((H, L, dk))
    Vh = rng.standard_normal((H, L, d))
    S = np.einsum("hid,hjd->hij", Q, K) / np.sqrt(dk)
    S = np.where(np.tril(np.ones((L, L), dtype=bool))[None], S, -np.inf)
    P = np.exp(S - S.max(axis=2, keepdims=True))
    P /= P.sum(axis=2, keepdims=True)
    Lp = -(-L // B) * B
    A = np.zeros((H, Lp, Lp), dtype=np.float32)
    A[:, :L, :L] = P.astype(np.float32)
    res = oracle.compress_seq(A, L, B, 1.0)
    V = np.ascontiguousarray(Vh.transpose(1, 0, 2)).astype(np.float32)  # [L, h_kv, d]
    O = oracle.retrieve_step(_bsr_of(res), B, np.eye(H, dtype=np.float32), V, H, [(L, L)], [0])
    ref_np = np.einsum("hij,jhd->ihd", A[:, :L, :L].astype(np.float64), V.astype(np.float64))
    np.testing.assert_allclose(O, ref_np, rtol=1e-10, atol=1e-12)
    sdpa = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q)[None], torch.from_numpy(K)[None],
        torch.from_numpy(V.astype(np.float64).transpose(1, 0, 2))[None], is_causal=True)[0]
    np.testing.assert_allclose(O, sdpa.permute(1, 0, 2).numpy(), rtol=2e-6, atol=2e-6)


def test_one_hot_W_and_gqa():
    L, B, h_s, h_r, h_kv, d = 30, 8, 3, 4, 2, 4
    A = smaps.gen_maps(L, B, h_s, 2, seed=9, dtype="f32")
    V = smaps.gen_v(L, h_kv, d, seed=9)
    res = oracle.compress_seq(A, L, B, 1.0)
    W = np.zeros((h_r, h_s), dtype=np.float32)
    src = [2, 0, 1, 2]
    for r, s in enumerate(src):
        W[r, s] = 1.0
    O = oracle.retrieve_step(_bsr_of(res), B, W, V, h_kv, [(L, L)], [0])
    An = np.where(causal_mask(L, A.shape[1])[None], A.numpy(), 0)[:, :L, :L].astype(np.float64)
    for r, s in enumerate(src):
        g = r // (h_r // h_kv)
        np.testing.assert_allclose(O[:, r, :], An[s] @ V.numpy()[:, g, :].astype(np.float64),
                                   rtol=1e-12, atol=1e-14)


def test_linear_in_W_and_V():
    L, B, h_s, h_r, h_kv, d = 33, 8, 2, 2, 1, 3
    A = smaps.gen_maps(L, B, h_s, 2, seed=4, dtype="f32")
    res = oracle.compress_seq(A, L, B, 0.9)
    # values on a 2**-10 grid, so W1 + W2 and V1 + V2 are exact in float32
    q = lambda x: np.round(np.asarray(x) * 1024.0).astype(np.float32) / np.float32(1024.0)
    W1 = q(smaps.gen_w(1, h_r, h_s, seed=1)[0].numpy())
    W2 = q(smaps.gen_w(1, h_r, h_s, seed=2)[0].numpy())
    V1 = q(smaps.gen_v(L, h_kv, d, seed=1).numpy())
    V2 = q(smaps.gen_v(L, h_kv, d, seed=2).numpy())
    f = lambda W, V: oracle.retrieve_step(_bsr_of(res), B, W, V, h_kv, [(L, L)], [0])
    np.testing.assert_allclose(f(W1 + W2, V1), f(W1, V1) + f(W2, V1), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(f(W1, V1 + V2), f(W1, V1) + f(W1, V2), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(f(-2 * W1, V1), -2 * f(W1, V1), rtol=1e-12, atol=1e-13)


def test_layouts_chunked_paged_varlen_identical():
    """Chunked prefill, a shuffled paged V and a varlen pack give the same O rows, bit for bit."""
    w = synth.Workload("t", (50, 29), B=8, h_s=2, h_r=2, h_kv=1, d=4, dtype="bf16", tau=0.9,
                       n_heavy=2, chunk=16, page_size=4)
    maps = [smaps.gen_maps(L, w.B, w.h_s, 2, seed=1, seq=s, dtype="bf16") for s, L in enumerate(w.lens)]
    row_ptr, col_idx, values, _ = oracle.compress_pack(maps, w.lens, w.B, w.tau)
    rows = lambda r: (col_idx[row_ptr[r]:row_ptr[r + 1]], values[row_ptr[r]:row_ptr[r + 1]])
    qbase = [0, w.nqb[0]]
    W = smaps.gen_w(1, w.h_r, w.h_s, seed=1)[0].numpy()
    T = sum(w.lens)
    V = smaps.gen_v(T, w.h_kv, w.d, seed=1, dtype="bf16")
    kst = [0, w.lens[0]]
    whole = oracle.retrieve_step(rows, w.B, W, V, w.h_kv, [(L, L) for L in w.lens], qbase, kst)
    # per-sequence calls
    per = [oracle.retrieve_step(rows, w.B, W, V, w.h_kv, [(L, L)], [qbase[s]], [kst[s]])
           for s, L in enumerate(w.lens)]
    assert np.array_equal(whole, np.concatenate(per, axis=0))
    # chunked
    parts = [[] for _ in w.lens]
    for step in synth.chunks(w):
        for s, (q, k) in enumerate(step):
            if q:
                parts[s].append(oracle.retrieve_step(rows, w.B, W, V, w.h_kv, [(q, k)], [qbase[s]], [kst[s]]))
    assert np.array_equal(whole, np.concatenate([np.concatenate(p, 0) for p in parts], 0))
    # paged
    table, npages = synth.page_table(w)
    Vp = torch.zeros((npages, w.page_size, w.h_kv, w.d), dtype=torch.bfloat16)
    for s, L in enumerate(w.lens):
        for t in range(L):
            Vp[table[s, t // w.page_size], t % w.page_size] = V[kst[s] + t]
    paged = oracle.retrieve_step(rows, w.B, W, Vp, w.h_kv, [(L, L) for L in w.lens], qbase,
                                 None, table, w.page_size)
    assert np.array_equal(whole, paged)
