"""Parity of the CUDA path (through the C ABI) with the CPU oracle, on the same seeded inputs.

Small cases compare every row; the full-size workloads compare sampled rows (the oracle
is run on the exact device bytes of each sampled row) plus layout identities that hold
at any size.  Block sets must match exactly except near-tie rows, which are counted and
expected to be 0; O must match within max-abs 2e-2 and relative-L2 1e-2 (bf16) or
1e-5 (float32).
"""
import numpy as np
import pytest
import torch

import cross_model_attention_mf_b200 as mf
import oracle
import synth
from synth import device as sdev
from tests.gpu_common import assert_O_close, check_rows, host_bsr, oracle_O_rows, run_compress

pytestmark = pytest.mark.gpu


def _retrieve(w, pack, bsr, W, V, force_simt=False, layer_map=(0,), layers=None):
    qbase = sdev.qblock_base(w)
    cu = pack.cu_seqlens
    return mf.mf_map_retrieve(layers or [bsr], list(layer_map), W, V, cu, cu, qbase, max(w.lens),
                              w.h_r, w.h_kv, total_q=w.tokens, force_simt=force_simt)


def _path(w, pack, bsr, W, V, force_simt=False):
    qbase = sdev.qblock_base(w)
    O = torch.empty((1, w.tokens, w.h_r, w.d), dtype=V.dtype, device=V.device)
    return mf.mf_retrieve_path([bsr], [0], W, V, pack.cu_seqlens, pack.cu_seqlens, qbase,
                               max(w.lens), w.h_r, w.h_kv, O, force_simt=force_simt)


def _status_ok():
    rc, bits = mf.mf_get_status()
    assert rc == mf.MF_OK and bits == 0, (rc, bits)


def _all_rows(w):
    return [(s, qb) for s in range(len(w.lens)) for qb in range(w.nqb[s])]


def _oracle_O_all(w, orows, W_l, V_host):
    outs = []
    starts = np.concatenate([[0], np.cumsum(w.lens)])
    for s in range(len(w.lens)):
        for qb in range(w.nqb[s]):
            O, _ = oracle_O_rows(w, orows, s, qb, W_l, V_host, 0, k_start=int(starts[s]))
            outs.append(O)
    return np.concatenate(outs, axis=0)


def _full_check(w, force_simt=False, expect_path=None):
    pack = sdev.fill_maps(sdev.alloc_maps(w), w, 0)
    bsr = run_compress(w, pack)
    _status_ok()
    orows, nb = check_rows(w, pack, bsr, _all_rows(w))
    if w.tau < 1.0:  # at tau = 1 every row ends exactly at tau: all rows are near-ties
        assert nb == 0
    W = sdev.w_weights(w)
    V = sdev.v_contiguous(w, 0)
    if expect_path is not None:
        assert _path(w, pack, bsr, W, V, force_simt) == expect_path
    O = _retrieve(w, pack, bsr, W, V, force_simt)
    _status_ok()
    want = _oracle_O_all(w, orows, W[0].cpu().numpy(), V.cpu())
    assert_O_close(O[0].float().cpu().numpy(), want, w.dtype, w.name)
    return pack, bsr, W, V, O


def test_gpu_generator_matches_cpu_recipe():
    for dt in ("f32", "bf16"):
        w = synth.Workload("g", (77, 40), B=32, h_s=3, h_r=1, h_kv=1, d=8, dtype=dt, tau=0.9, n_heavy=5)
        pack = sdev.fill_maps(sdev.alloc_maps(w), w, 2)
        for s, L in enumerate(w.lens):
            g = pack.seq_view(s, w.h_s, w.B).float().cpu().numpy()
            c = synth.gen_maps(L, w.B, w.h_s, 5, seed=0, layer=2, seq=s, dtype=dt).float().numpy()
            Lp = c.shape[1]
            causal = np.tril(np.ones((Lp, Lp), dtype=bool))
            if dt == "f32":
                np.testing.assert_allclose(g[:, causal], c[:, causal], rtol=2e-5, atol=1e-7)
            else:  # at most one bf16 rounding step apart
                np.testing.assert_allclose(g[:, causal], c[:, causal], rtol=2 ** -7, atol=1e-8)


def test_tiny_fp32():
    w = synth.ALL["tiny"]
    _full_check(w, expect_path=0)


def test_small_bf16_varlen_tcgen05():
    w = synth.Workload("small", (300, 129, 64, 1), B=64, h_s=32, h_r=32, h_kv=8, d=128,
                       dtype="bf16", tau=0.95, n_heavy=16, reading=3)
    pack, bsr, W, V, O = _full_check(w, expect_path=1)
    # the SIMT kernel on the same BSR agrees with the tensor-core kernel
    O2 = _retrieve(w, pack, bsr, W, V, force_simt=True)
    _status_ok()
    assert_O_close(O[0].float().cpu().numpy(), O2[0].float().cpu().numpy(), "bf16", "tc vs simt")


@pytest.mark.parametrize("nseq", [64, 70])
def test_many_sequences(nseq):
    """A batch of short sequences around the 64-sequence limit of the geometry computed inside
    the statistics kernel (64: inside, 70: the separate geometry pass); ~200 query blocks, so
    the selection's look-back runs over several 32-row windows.  Every row's kept set, values
    and O are compared with the oracle."""
    lens = tuple(64 + (37 * k) % 257 for k in range(nseq))
    w = synth.Workload(f"many{nseq}", lens, B=64, h_s=16, h_r=16, h_kv=4, d=128, dtype="bf16",
                       tau=0.95, n_heavy=8, reading=3)
    assert sum(w.nqb) > 64
    _full_check(w, expect_path=1)


def test_small_bf16_simt_path():
    w = synth.Workload("small_simt", (200, 70), B=64, h_s=32, h_r=32, h_kv=8, d=128,
                       dtype="bf16", tau=0.9, n_heavy=16, reading=3)
    _full_check(w, force_simt=True, expect_path=0)


def test_long_block_gqa3_tcgen05():
    w = synth.Workload("b128", (400, 130), B=128, h_s=32, h_r=24, h_kv=8, d=128, dtype="bf16",
                       tau=0.9, n_heavy=8, reading=3)
    _full_check(w, expect_path=1)


def test_qwen_heads_40_tcgen05():
    w = synth.Workload("hs40", (200, 77, 130), B=64, h_s=40, h_r=32, h_kv=8, d=128, dtype="bf16",
                       tau=0.95, n_heavy=16, reading=3)
    _full_check(w, expect_path=1)


def test_uneven_kv_groups_tcgen05():
    """h_kv = 6: the second head chunk holds two real groups and two empty ones."""
    w = synth.Workload("kv6", (150,), B=64, h_s=16, h_r=12, h_kv=6, d=128, dtype="bf16",
                       tau=0.9, n_heavy=4, reading=3)
    _full_check(w, expect_path=1)


@pytest.mark.parametrize("tau", [0.0, 1.0])
def test_tau_extremes(tau):
    w = synth.Workload("tau", (260,), B=64, h_s=8, h_r=8, h_kv=2, d=128, dtype="bf16", tau=tau,
                       n_heavy=4, reading=3)
    pack, bsr, W, V, O = _full_check(w, expect_path=1)
    rp, ci, nnz = host_bsr(bsr)
    if tau == 0.0:
        assert nnz == w.nqb[0] and ci[:nnz].tolist() == list(range(w.nqb[0]))
    else:
        # tau = 1: O equals the dense receiver map times V (numpy, float64)
        A = pack.seq_view(0, w.h_s, w.B).float().cpu().numpy().astype(np.float64)
        L = w.lens[0]
        A = np.tril(A[:, :L, :L])
        P = np.einsum("rs,sij->rij", W[0].cpu().numpy().astype(np.float64), A)
        Vr = np.repeat(V.float().cpu().numpy().astype(np.float64), w.h_r // w.h_kv, axis=1)
        dense = np.einsum("rij,jrd->ird", P, Vr)
        assert_O_close(O[0].float().cpu().numpy(), dense, "bf16", "tau=1 vs dense")


def test_identity_W_is_causal_attention():
    """W = I, maps = causal softmax(Q K^T / sqrt(dk)) stored in bf16, tau = 1: O is standard
    causal attention (torch SDPA on the same Q, K, V)."""
    torch.manual_seed(0)
    H, L, B, dk = 8, 200, 64, 64
    Q = torch.randn(H, L, dk, dtype=torch.float64)
    K = torch.randn(H, L, dk, dtype=torch.float64)
    Vh = torch.randn(L, H, 128, dtype=torch.float64)
    S = torch.einsum("hid,hjd->hij", Q, K) / dk ** 0.5
    S = S.masked_fill(~torch.tril(torch.ones(L, L, dtype=torch.bool)), float("-inf"))
    Pm = torch.softmax(S, dim=-1)
    Lp = 256
    w = synth.Workload("qk", (L,), B=B, h_s=H, h_r=H, h_kv=H, d=128, dtype="bf16", tau=1.0, n_heavy=0)
    pack = sdev.alloc_maps(w)
    view = pack.seq_view(0, H, B)
    view.zero_()
    view[:, :L, :L] = Pm.to(torch.bfloat16).cuda()
    bsr = run_compress(w, pack)
    W = torch.eye(H, dtype=torch.float32, device="cuda")[None]
    V = Vh.to(torch.bfloat16).cuda()
    O = _retrieve(w, pack, bsr, W, V)
    _status_ok()
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q[None], K[None], Vh.to(torch.bfloat16).double().permute(1, 0, 2)[None], is_causal=True)[0]
    assert_O_close(O[0].float().cpu().numpy(), ref.permute(1, 0, 2).numpy(), "bf16", "W=I vs SDPA")


def test_layouts_bitwise_identical():
    """Chunked prefill over a shuffled paged V, a contiguous V, one call per sequence and the
    varlen pack all give bit-identical O rows on the tensor-core path."""
    w = synth.Workload("lay", (700, 333, 64), B=64, h_s=32, h_r=32, h_kv=8, d=128, dtype="bf16",
                       tau=0.95, n_heavy=16, reading=3, chunk=256, page_size=16)
    pack = sdev.fill_maps(sdev.alloc_maps(w), w, 0)
    bsr = run_compress(w, pack)
    W = sdev.w_weights(w)
    V = sdev.v_contiguous(w, 0)
    whole = _retrieve(w, pack, bsr, W, V)[0]
    qbase = sdev.qblock_base(w)
    starts = np.concatenate([[0], np.cumsum(w.lens)])
    # per-sequence calls
    for s, L in enumerate(w.lens):
        cu = torch.tensor([0, L], dtype=torch.int32, device="cuda")
        Os = mf.mf_map_retrieve([bsr], [0], W, V[starts[s]:starts[s] + L].contiguous(), cu, cu,
                                qbase[s:s + 1].contiguous(), L, w.h_r, w.h_kv, total_q=L)[0]
        assert torch.equal(Os, whole[starts[s]:starts[s] + L])
    # paged, whole sequences
    Vp, table = sdev.v_paged(w, V)
    cu = pack.cu_seqlens
    paged = mf.mf_map_retrieve([bsr], [0], W, Vp, cu, cu, qbase, max(w.lens), w.h_r, w.h_kv,
                               total_q=w.tokens, paged=(table, w.page_size))[0]
    assert torch.equal(paged, whole)
    # chunked prefill, paged
    parts = [[] for _ in w.lens]
    for step in synth.chunks(w):
        cu_q, cu_k, mq = sdev.step_tensors(step)
        Oc = mf.mf_map_retrieve([bsr], [0], W, Vp, cu_q, cu_k, qbase, mq, w.h_r, w.h_kv,
                                total_q=int(cu_q[-1]), paged=(table, w.page_size))[0]
        q = cu_q.cpu().numpy()
        for s in range(len(w.lens)):
            if q[s + 1] > q[s]:
                parts[s].append(Oc[q[s]:q[s + 1]])
    chunked = torch.cat([torch.cat(p) for p in parts])
    assert torch.equal(chunked, whole)
    # chunked prefill, contiguous prefixes
    for step in synth.chunks(w)[:2]:
        cu_q, cu_k, mq = sdev.step_tensors(step)
        Vc = sdev.pack_prefixes(V, w.lens, step)
        Oc = mf.mf_map_retrieve([bsr], [0], W, Vc, cu_q, cu_k, qbase, mq, w.h_r, w.h_kv,
                                total_q=int(cu_q[-1]))[0]
        Op = mf.mf_map_retrieve([bsr], [0], W, Vp, cu_q, cu_k, qbase, mq, w.h_r, w.h_kv,
                                total_q=int(cu_q[-1]), paged=(table, w.page_size))[0]
        assert torch.equal(Oc, Op)
    _status_ok()


@pytest.mark.parametrize("page_size", [8, 16, 32, 64])
def test_paged_page_sizes_bitwise(page_size):
    """Every supported page size (the V slot holds whole pages of both groups of a half tile, a
    K step of 16 keys spanning two 8-token pages or part of a larger one) gives O bit for bit
    equal to contiguous V."""
    w = synth.Workload(f"pg{page_size}", (300, 129, 64), B=64, h_s=32, h_r=32, h_kv=8, d=128,
                       dtype="bf16", tau=0.95, n_heavy=16, reading=3, page_size=page_size)
    pack = sdev.fill_maps(sdev.alloc_maps(w), w, 0)
    bsr = run_compress(w, pack)
    W = sdev.w_weights(w)
    V = sdev.v_contiguous(w, 0)
    whole = _retrieve(w, pack, bsr, W, V)[0]
    Vp, table = sdev.v_paged(w, V)
    cu = pack.cu_seqlens
    paged = mf.mf_map_retrieve([bsr], [0], W, Vp, cu, cu, sdev.qblock_base(w), max(w.lens),
                               w.h_r, w.h_kv, total_q=w.tokens, paged=(table, w.page_size))[0]
    _status_ok()
    assert torch.equal(paged, whole)


@pytest.mark.parametrize("h_r,h_kv", [(4, 1), (8, 2), (12, 3)])
def test_few_kv_heads_tcgen05(h_r, h_kv):
    """One, two and three KV heads on the tensor-core path (the V copies hold two heads, or one
    when there is only one) against the oracle."""
    w = synth.Workload(f"kv{h_kv}", (300, 129), B=64, h_s=16, h_r=h_r, h_kv=h_kv, d=128,
                       dtype="bf16", tau=0.95, n_heavy=8, reading=3)
    _full_check(w, expect_path=1)


def test_layer_batch_and_layer_map():
    """Three receiver layers over two sender layers in one call equal three single-layer calls."""
    w = synth.Workload("lm", (200,), B=64, h_s=32, h_r=32, h_kv=8, d=128, dtype="bf16", tau=0.9,
                       n_heavy=8, reading=3, n_sender_layers=2, n_receiver_layers=3)
    bsrs = []
    for l in range(2):
        pack = sdev.fill_maps(sdev.alloc_maps(w), w, l)
        bsrs.append(run_compress(w, pack))
    W = sdev.w_weights(w)
    V = torch.stack([sdev.v_contiguous(w, l) for l in range(3)])
    lm = [0, 1, 1]
    qbase = sdev.qblock_base(w)
    cu = pack.cu_seqlens
    Oall = mf.mf_map_retrieve(bsrs, lm, W, V, cu, cu, qbase, 200, w.h_r, w.h_kv, total_q=200,
                              v_layer_stride=V[0].numel())
    for l in range(3):
        Ol = mf.mf_map_retrieve(bsrs, lm, W, V, cu, cu, qbase, 200, w.h_r, w.h_kv, total_q=200,
                                l_r_range=(l, l + 1), v_layer_stride=V[0].numel())
        assert torch.equal(Ol[0], Oall[l])
    assert not torch.equal(Oall[0], Oall[1])
    _status_ok()


# ------------------------------------------------------------------ device-side error reporting

def test_capacity_overflow_reported():
    w = synth.Workload("cap", (300,), B=64, h_s=8, h_r=8, h_kv=2, d=128, dtype="bf16", tau=0.99,
                       n_heavy=4, reading=3)
    pack = sdev.fill_maps(sdev.alloc_maps(w), w, 0)
    full = run_compress(w, pack)
    _status_ok()
    n = int(full.nnz.cpu()[0])
    small = run_compress(w, pack, capacity=n - 2)
    rc, bits = mf.mf_get_status()
    assert rc == mf.MF_ERR_CAPACITY and bits & 2
    assert int(small.nnz.cpu()[0]) == n
    assert torch.equal(small.col_idx[:n - 2], full.col_idx[:n - 2])
    assert torch.equal(small.values[:n - 2], full.values[:n - 2])


@pytest.mark.parametrize("force_simt", [False, True])
def test_bad_bsr_index_reported_not_faulted(force_simt):
    w = synth.Workload("bad", (200,), B=64, h_s=32, h_r=32, h_kv=8, d=128, dtype="bf16", tau=0.9,
                       n_heavy=8, reading=3)
    pack = sdev.fill_maps(sdev.alloc_maps(w), w, 0)
    bsr = run_compress(w, pack)
    W = sdev.w_weights(w)
    V = sdev.v_contiguous(w, 0)
    _status_ok()
    bsr.col_idx[0] = 7  # row 0 may only reference key block 0
    _retrieve(w, pack, bsr, W, V, force_simt=force_simt)
    rc, bits = mf.mf_get_status()
    assert rc == mf.MF_ERR_DEVICE_INDEX and bits & 1
    bsr.row_ptr[1] = 1 << 30  # a row pointer beyond capacity: the row is skipped
    _retrieve(w, pack, bsr, W, V, force_simt=force_simt)
    rc, bits = mf.mf_get_status()
    assert rc == mf.MF_ERR_DEVICE_INDEX
    torch.cuda.synchronize()


def test_bad_page_reported():
    w = synth.Workload("page", (200,), B=64, h_s=32, h_r=32, h_kv=8, d=128, dtype="bf16", tau=0.9,
                       n_heavy=8, reading=3, page_size=16)
    pack = sdev.fill_maps(sdev.alloc_maps(w), w, 0)
    bsr = run_compress(w, pack)
    V = sdev.v_contiguous(w, 0)
    Vp, table = sdev.v_paged(w, V)
    table[0, 3] = 10 ** 6
    cu = pack.cu_seqlens
    mf.mf_map_retrieve([bsr], [0], sdev.w_weights(w), Vp, cu, cu, sdev.qblock_base(w), 200,
                       w.h_r, w.h_kv, total_q=200, paged=(table, 16))
    rc, bits = mf.mf_get_status()
    assert rc == mf.MF_ERR_DEVICE_INDEX and bits & 16


@pytest.mark.parametrize("entry", ["mf_compress", "mf_compress_static"])
def test_empty_batch(entry):
    """A batch with no query block (max_seqlen 0, an empty sequence) is valid input: an empty
    BSR (row_ptr [0], nnz 0) and nothing else; retrieval over it writes nothing."""
    import ctypes
    dev = "cuda"
    maps = torch.zeros(8, dtype=torch.bfloat16, device=dev)
    off = torch.zeros(1, dtype=torch.int64, device=dev)
    cu = torch.zeros(2, dtype=torch.int32, device=dev)
    out = mf.alloc_bsr(0, 4, 4, 64, torch.bfloat16, dev)
    out.row_ptr.fill_(-7)
    out.nnz.fill_(-7)
    if entry == "mf_compress":
        mf.mf_compress(maps, off, cu, 0, 4, 64, 0.9, out)
    else:
        d = mf._compress_desc(maps, off, cu, 0, 4, 64, 0.9, out)
        assert mf._lib.mf_compress_static(ctypes.byref(d), torch.cuda.current_stream().cuda_stream) == mf.MF_OK
    _status_ok()
    assert out.row_ptr.cpu().tolist() == [0] and int(out.nnz.cpu()[0]) == 0
    W = torch.zeros((1, 4, 4), dtype=torch.float32, device=dev)
    V = torch.zeros((1, 1, 128), dtype=torch.bfloat16, device=dev)
    O = torch.full((1, 1, 4, 128), 3.0, dtype=torch.bfloat16, device=dev)
    qb = torch.zeros(1, dtype=torch.int32, device=dev)
    mf.mf_map_retrieve([out], [0], W, V, cu, cu, qb, 0, 4, 1, O=O)
    _status_ok()
    assert (O == 3.0).all()


def _raw_close(got, want, amax, rl2, what):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = float(np.abs(got - want).max())
    rel = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30))
    print(f"[O f32] {what}: raw max-abs {err:.3e}, rel-L2 {rel:.3e}")
    assert err <= amax and rel <= rl2, f"{what}: raw max-abs {err:.3e} (<= {amax}), rel-L2 {rel:.3e} (<= {rl2})"


@pytest.mark.parametrize("name,lens,B,h_s,h_r,h_kv,reading", [
    ("f32out_varlen", (300, 129, 64), 64, 32, 32, 8, 3),
    ("f32out_b128_gq3", (400,), 128, 32, 24, 8, 3),
    ("f32out_hs40", (257,), 64, 40, 32, 8, 1),
])
def test_float32_output_meets_the_literal_bounds(name, lens, B, h_s, h_r, h_kv, reading):
    """With float32 O (MF_RETRIEVE_O_F32) the tensor-core kernel's accumulators are compared
    with the oracle unrounded: raw max-abs 2e-2 and relative L2 1e-2, every row.  With P as a
    bf16 pair everywhere (MF_RETRIEVE_P_SPLIT) the bf16 output is that float32 output rounded
    to nearest even, bit for bit; by default the same holds in the first query block of each
    sequence (P split there), and every row meets the bf16 bounds."""
    w = synth.Workload(name, lens, B=B, h_s=h_s, h_r=h_r, h_kv=h_kv, d=128, dtype="bf16", tau=0.95,
                       n_heavy=16, reading=reading)
    pack = sdev.fill_maps(sdev.alloc_maps(w), w, 0)
    bsr = run_compress(w, pack)
    _status_ok()
    orows, _ = check_rows(w, pack, bsr, _all_rows(w))
    W = sdev.w_weights(w)
    V = sdev.v_contiguous(w, 0)
    qbase, cu = sdev.qblock_base(w), pack.cu_seqlens
    O32 = mf.mf_map_retrieve([bsr], [0], W, V, cu, cu, qbase, max(w.lens), w.h_r, w.h_kv,
                             total_q=w.tokens, o_f32=True)[0]
    O16 = mf.mf_map_retrieve([bsr], [0], W, V, cu, cu, qbase, max(w.lens), w.h_r, w.h_kv,
                             total_q=w.tokens)[0]
    _status_ok()
    O16s = mf.mf_map_retrieve([bsr], [0], W, V, cu, cu, qbase, max(w.lens), w.h_r, w.h_kv,
                              total_q=w.tokens, p_split=True)[0]
    _status_ok()
    assert O32.dtype == torch.float32
    R32 = O32.to(torch.bfloat16)
    assert torch.equal(R32, O16s)
    starts = np.concatenate([[0], np.cumsum(w.lens)])
    for s0, L in zip(starts[:-1], w.lens):
        first = slice(int(s0), int(s0) + min(B, L))
        assert torch.equal(R32[first], O16[first]), "first query block: P split"
    want = _oracle_O_all(w, orows, W[0].cpu().numpy(), V.cpu())
    _raw_close(O32.cpu().numpy(), want, 2e-2, 1e-2, name)
    assert_O_close(O16.float().cpu().numpy(), want, "bf16", f"{name} bf16 output")


def test_float32_output_full_size_sampled():
    """The Ministral-like pair with float32 O: sampled query blocks held to the literal bounds."""
    w = synth.ALL["ministral_pair"]
    pack = sdev.fill_maps(sdev.alloc_maps(w), w, 0)
    bsr = run_compress(w, pack)
    _status_ok()
    rows = [(0, qb) for qb in (0, 1, 63, 64, 126, 127)]
    orows, nb = check_rows(w, pack, bsr, rows)
    assert nb == 0
    W = sdev.w_weights(w)
    V = sdev.v_contiguous(w, 0)
    cu = pack.cu_seqlens
    O = mf.mf_map_retrieve([bsr], [0], W, V, cu, cu, sdev.qblock_base(w), w.lens[0], w.h_r,
                           w.h_kv, total_q=w.tokens, o_f32=True)[0]
    _status_ok()
    Wl, Vh = W[0].cpu().numpy(), V.cpu()
    for _, qb in rows:
        want, (lo, hi) = oracle_O_rows(w, orows, 0, qb, Wl, Vh, 0)
        _raw_close(O[qb * w.B + lo:qb * w.B + hi].cpu().numpy(), want, 2e-2, 1e-2, f"ministral qb={qb}")
    del pack, bsr, O
    torch.cuda.empty_cache()


def test_float32_output_refused_on_the_simt_path():
    w = synth.ALL["tiny"]
    pack = sdev.fill_maps(sdev.alloc_maps(w), w, 0)
    bsr = run_compress(w, pack)
    W, V = sdev.w_weights(w), sdev.v_contiguous(w, 0)
    cu = pack.cu_seqlens
    with pytest.raises(mf.MFError) as e:
        mf.mf_map_retrieve([bsr], [0], W, V, cu, cu, sdev.qblock_base(w), w.lens[0], w.h_r, w.h_kv,
                           total_q=w.tokens, o_f32=True)
    assert e.value.status == mf.MF_ERR_UNSUPPORTED
    _status_ok()
