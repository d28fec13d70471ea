"""Parity of compression straight from Q, K (mf_compress_qk, tcgen05) with the oracle.

The oracle computes the sender's causal attention maps in float64 from the exact bf16 bytes
of Q and K, then the same block statistics, selection and gather as for dense maps.  Checks:
  - block masses within 1e-5 relative (float32 exp-sums combined in float64 on the GPU);
  - kept sets identical, except near-tie rows (oracle.is_boundary), whose GPU set must still
    be a valid selection on the oracle's masses;
  - kept values within a bf16 rounding (2^-8 relative) plus 1e-5 relative and 1e-7 absolute;
  - the row log2-sum-exp within 1e-4 of torch.logsumexp in float64.
"""
import math

import numpy as np
import pytest
import torch

import cross_model_attention_mf_b200 as mf
import oracle
from synth.qk import gen_qk

pytestmark = pytest.mark.gpu

B, D = 64, 128


def _status(expect=0):
    rc, bits = mf.mf_get_status()
    assert bits == expect, (rc, bits)


def _run(lens, h_s, h_kv, tau, n_heavy=8, seed=0, capacity=None, scale=0.0):
    Q, K = gen_qk(lens, h_s, h_kv, D, n_heavy, seed)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    nqb = [-(-L // B) for L in lens]
    causal = sum(n * (n + 1) // 2 for n in nqb)
    cap = causal if capacity is None else capacity
    out = mf.alloc_bsr(sum(nqb), cap, h_s, B, torch.bfloat16, "cuda", n_causal=causal)
    lse = torch.full((h_s, sum(lens)), float("nan"), dtype=torch.float32, device="cuda")
    mf.mf_compress_qk(Q.cuda(), K.cuda(), cu, max(lens), B, tau, out, scale=scale, lse=lse)
    return Q, K, out, lse, nqb


def _check(lens, h_s, h_kv, tau, rows=None, **kw):
    Q, K, out, lse, nqb = _run(lens, h_s, h_kv, tau, **kw)
    _status()
    scale = kw.get("scale", 0.0) or 1.0 / math.sqrt(D)
    rp = out.row_ptr.cpu().numpy()
    ci = out.col_idx.cpu().numpy()
    mass = out.block_mass.cpu().numpy()
    nnz = int(out.nnz.cpu()[0])
    assert rp[-1] == nnz
    starts = np.concatenate([[0], np.cumsum(lens)])
    row_base = np.concatenate([[0], np.cumsum(nqb)])
    cb_base = np.concatenate([[0], np.cumsum([n * (n + 1) // 2 for n in nqb])])
    todo = rows if rows is not None else [(s, qb) for s in range(len(lens)) for qb in range(nqb[s])]
    nb = 0
    for s, qb in todo:
        L = lens[s]
        Qs, Ks = Q[starts[s]:starts[s] + L], K[starts[s]:starts[s] + L]
        m, kept, info, vals = oracle.compress_qk_row(Qs, Ks, L, B, qb, tau, scale)
        gm = mass[cb_base[s] + qb * (qb + 1) // 2:][:qb + 1]
        np.testing.assert_allclose(gm, m, rtol=1e-5, atol=1e-9, err_msg=f"masses s={s} qb={qb}")
        r = row_base[s] + qb
        g = ci[rp[r]:rp[r + 1]]
        if oracle.is_boundary(info, tau):
            nb += 1
            assert g.tolist() == sorted(g.tolist()) and qb in g.tolist()
            assert m[g].sum() >= tau * m.sum() * (1 - 1e-5)
            continue
        assert g.tolist() == kept.tolist(), f"kept s={s} qb={qb}: gpu {g} oracle {kept}"
        gv = out.values[rp[r]:rp[r + 1]].double().cpu().numpy()
        err = np.abs(gv - vals) - (2.0 ** -8 + 1e-5) * np.abs(vals)
        assert err.max() <= 1e-7, f"values s={s} qb={qb}: excess {err.max():.3e}"
        # row log2-sum-exp against torch in float64
        i0, i1 = qb * B, min(L, (qb + 1) * B)
        q = Qs[i0:i1].double().permute(1, 0, 2)                          # [h_s, rows, d]
        k = Ks[:i1].double().repeat_interleave(h_s // h_kv, dim=1).permute(1, 0, 2)
        sc = scale * q @ k.transpose(1, 2)
        causal = torch.arange(i1)[None, :] <= torch.arange(i0, i1)[:, None]
        want = torch.logsumexp(sc.masked_fill(~causal, -math.inf), dim=2) / math.log(2.0)
        got = lse[:, starts[s] + i0:starts[s] + i1].double().cpu()
        torch.testing.assert_close(got, want, rtol=0, atol=1e-4)
    return out, nb, nnz


def test_small_varlen_gqa():
    out, nb, _ = _check((300, 129, 64, 1), 8, 2, 0.95)
    assert nb == 0


def test_ragged_mha_and_scale():
    out, nb, _ = _check((200, 65, 127, 128), 3, 3, 0.9, scale=0.05)
    assert nb == 0


@pytest.mark.parametrize("tau", [0.0, 1.0])
def test_tau_extremes(tau):
    lens = (257, 70)
    out, nb, nnz = _check(lens, 4, 1, tau)
    nqb = [-(-L // B) for L in lens]
    if tau == 0.0:
        assert nnz == sum(nqb)                                      # the diagonal only
    else:
        assert nnz == sum(n * (n + 1) // 2 for n in nqb)            # every causal block


def test_capacity_overflow_reported():
    Q, K, out, lse, nqb = _run((400,), 4, 2, 1.0, capacity=5)
    rc, bits = mf.mf_get_status()
    assert bits == 2 and rc == mf.MF_ERR_CAPACITY
    assert int(out.nnz.cpu()[0]) == 7 * 8 // 2


def test_full_size_ministral_like_sampled_rows():
    """One 8192-token sequence, 32 query heads over 8 key heads: sampled rows against the
    oracle (each row's float64 maps computed from the device's exact Q, K bytes)."""
    out, nb, nnz = _check((8192,), 32, 8, 0.95, n_heavy=16,
                          rows=[(0, 0), (0, 1), (0, 37), (0, 100), (0, 127)])
    assert nb == 0
    assert 0 < nnz < 128 * 129 // 2
