"""Stored reference values for the tiny workload (tests/golden/tiny_oracle.json).

The MapFlow pages print no worked example, so the stored values come from the oracle
(tests/golden/make_golden.py, which calls only `synth` for the inputs and `oracle/`).  The CPU
test pins the oracle against drift; the GPU test checks the CUDA path against the stored file
on the exact same host-generated input bytes.
"""
import json
import os
import sys

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
GOLD = os.path.join(HERE, "golden", "tiny_oracle.json")
sys.path.insert(0, os.path.join(HERE, "golden"))


def _stored():
    with open(GOLD) as f:
        return json.load(f)


def test_oracle_reproduces_stored_tiny_values():
    import make_golden
    got, want = make_golden.compute(), _stored()
    assert got["row_ptr"] == want["row_ptr"]
    assert got["col_idx"] == want["col_idx"]
    for a, b in zip(got["block_mass"], want["block_mass"]):
        np.testing.assert_allclose(a, b, rtol=1e-14, atol=0)
    assert got["O_rows"] == want["O_rows"] and got["O_shape"] == want["O_shape"]
    np.testing.assert_allclose(got["O_sampled"], want["O_sampled"], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose([got["O_sum"], got["O_sumsq"]], [want["O_sum"], want["O_sumsq"]],
                               rtol=1e-12)


def test_stored_tiny_selection_is_well_formed():
    want = _stored()
    rp, ci = want["row_ptr"], want["col_idx"]
    assert rp[0] == 0 and len(rp) == 9 and rp[-1] == len(ci)
    for qb in range(8):
        row = ci[rp[qb]:rp[qb + 1]]
        assert row == sorted(set(row)) and qb in row and all(0 <= kb <= qb for kb in row)


@pytest.mark.gpu
def test_cuda_path_matches_stored_tiny_values():
    import torch
    import cross_model_attention_mf_b200 as mf
    import synth
    from synth import device as sdev
    from gpu_common import assert_O_close

    want = _stored()
    w = synth.ALL["tiny"]
    L = w.lens[0]
    pack = sdev.fill_maps(sdev.alloc_maps(w), w, 0, use_gpu=False)
    W = sdev.w_weights(w)
    V = sdev.v_contiguous(w, 0, use_gpu=False)
    bsr = mf.alloc_bsr(sum(w.nqb), w.causal_blocks, w.h_s, w.B, pack.maps.dtype, "cuda",
                       n_causal=w.causal_blocks)
    mf.mf_compress(pack.maps, pack.map_seq_offset, pack.cu_seqlens, L, w.h_s, w.B, w.tau, bsr)
    O = torch.empty((1, L, w.h_r, w.d), dtype=torch.float32, device="cuda")
    cu = pack.cu_seqlens
    mf.mf_map_retrieve([bsr], [0], W, V, cu, cu, sdev.qblock_base(w), L, w.h_r, w.h_kv, O=O)
    rc, bits = mf.mf_get_status()
    assert rc == mf.MF_OK and bits == 0
    n = int(bsr.nnz.cpu()[0])
    assert bsr.row_ptr.cpu().tolist() == want["row_ptr"]
    assert bsr.col_idx[:n].cpu().tolist() == want["col_idx"]
    mass = bsr.block_mass.cpu().numpy()
    flat = np.concatenate([np.asarray(m) for m in want["block_mass"]])
    np.testing.assert_allclose(mass, flat, rtol=2e-6, atol=1e-12)
    got = O[0].cpu().numpy()[want["O_rows"]].reshape(-1)
    assert_O_close(got, np.asarray(want["O_sampled"]), "f32", "tiny vs stored")


GOLD_QK = os.path.join(HERE, "golden", "tiny_qk_oracle.json")


def _stored_qk():
    with open(GOLD_QK) as f:
        return json.load(f)


def test_oracle_reproduces_stored_qk_values():
    import make_golden
    got, want = make_golden.compute_qk(), _stored_qk()
    assert len(got["rows"]) == len(want["rows"])
    for a, b in zip(got["rows"], want["rows"]):
        assert a["kept"] == b["kept"]
        np.testing.assert_allclose(a["mass"], b["mass"], rtol=1e-13, atol=0)
        np.testing.assert_allclose(a["vals_sampled"], b["vals_sampled"], rtol=1e-11, atol=1e-15)
        np.testing.assert_allclose(a["vals_sum"], b["vals_sum"], rtol=1e-12)


@pytest.mark.gpu
def test_gpu_compress_qk_matches_stored_values():
    import torch
    import cross_model_attention_mf_b200 as mf
    import make_golden
    import oracle
    want = _stored_qk()["rows"]
    Q, K = make_golden.qk_case()
    lens, B, tau = make_golden.QK_LENS, make_golden.QK_B, make_golden.QK_TAU
    nqb = [-(-L // B) for L in lens]
    causal = sum(n * (n + 1) // 2 for n in nqb)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    out = mf.alloc_bsr(sum(nqb), causal, make_golden.QK_HS, B, torch.bfloat16, "cuda", n_causal=causal)
    mf.mf_compress_qk(Q.cuda(), K.cuda(), cu, max(lens), B, tau, out)
    rc, bits = mf.mf_get_status()
    assert bits == 0
    rp, ci = out.row_ptr.cpu().numpy(), out.col_idx.cpu().numpy()
    mass = out.block_mass.cpu().numpy()
    row, cb = 0, 0
    for n in nqb:
        for qb in range(n):
            w = want[row]
            np.testing.assert_allclose(mass[cb:cb + qb + 1], w["mass"], rtol=1e-5, atol=1e-9)
            _, info = oracle.select(np.array(w["mass"]), qb, tau)
            if not oracle.is_boundary(info, tau):
                assert ci[rp[row]:rp[row + 1]].tolist() == w["kept"]
                gsum = out.values[rp[row]:rp[row + 1]].double().sum().item()
                np.testing.assert_allclose(gsum, w["vals_sum"], rtol=2e-3)
            row += 1
            cb += qb + 1
