"""The bounded waits of the tensor-core kernels: a wait that runs out is reported, and the
device stays usable.

Every pipeline wait in k_retrieve_tc, k_qk and k_calib_gram_tc gives up after a time limit:
the CTA records MF_ERR_TIMEOUT, all its roles stop, the copies and MMAs it issued are waited
for and its tensor memory is released.  mf_set_wait_limit(limit, stall=True) makes the MMA
warp of every CTA first wait on a barrier that nothing arrives at, so the limit is certain to
run out, without a fault and without a hang.  Each test then checks the status word, and that
a normal call afterwards reproduces, bit for bit, the result of a call made before the stall
(a CTA that left tensor memory allocated or copies in flight would break the later call).
"""
import numpy as np
import pytest
import torch

import cross_model_attention_mf_b200 as mf
import synth
from synth import device as sdev
from tests.gpu_common import run_compress

pytestmark = pytest.mark.gpu

LIMIT_NS = 20_000_000  # 20 ms


def _stalled(fn):
    """Run fn with the stall on; return the status it leaves."""
    torch.cuda.synchronize()
    rc0, _ = mf.mf_get_status()
    assert rc0 == mf.MF_OK
    mf.mf_set_wait_limit(LIMIT_NS, stall=True)
    try:
        fn()
        rc, bits = mf.mf_get_status()
    finally:
        mf.mf_set_wait_limit(0, stall=False)
    return rc, bits


def _clean():
    rc, bits = mf.mf_get_status()
    assert rc == mf.MF_OK and bits == 0, (rc, bits)


def test_retrieve_timeout_then_clean_call():
    w = synth.Workload("stall", (700,), B=64, h_s=32, h_r=32, h_kv=8, d=128, dtype="bf16",
                       tau=0.95, n_heavy=16, reading=3)
    pack = sdev.fill_maps(sdev.alloc_maps(w), w, 0)
    bsr = run_compress(w, pack)
    W, V, qb, cu = sdev.w_weights(w), sdev.v_contiguous(w, 0), sdev.qblock_base(w), pack.cu_seqlens

    def call():
        return mf.mf_map_retrieve([bsr], [0], W, V, cu, cu, qb, 700, w.h_r, w.h_kv, total_q=700)[0]

    assert mf.mf_retrieve_path([bsr], [0], W, V, cu, cu, qb, 700, w.h_r, w.h_kv,
                               torch.empty((1, 700, 32, 128), dtype=torch.bfloat16, device="cuda")) == 1
    ref = call()
    _clean()
    rc, bits = _stalled(call)
    assert rc == mf.MF_ERR_TIMEOUT and bits & 4, (rc, bits)
    again = call()
    _clean()
    assert torch.equal(again, ref)


def test_compress_qk_timeout_then_clean_call():
    from synth.qk import gen_qk
    lens, h_s, h_kv, B, tau = (300, 77), 8, 2, 64, 0.95
    Q, K = gen_qk(lens, h_s, h_kv, 128, 8, 0)
    Q, K = Q.cuda(), K.cuda()
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    nqb = [-(-L // B) for L in lens]
    ncb = sum(n * (n + 1) // 2 for n in nqb)

    def call():
        out = mf.alloc_bsr(sum(nqb), ncb, h_s, B, torch.bfloat16, "cuda", n_causal=ncb)
        mf.mf_compress_qk(Q, K, cu, max(lens), B, tau, out)
        return out

    ref = call()
    _clean()
    rc, bits = _stalled(call)
    assert rc == mf.MF_ERR_TIMEOUT and bits & 4, (rc, bits)
    again = call()
    _clean()
    n = int(ref.nnz.cpu()[0])
    assert int(again.nnz.cpu()[0]) == n
    assert torch.equal(again.row_ptr, ref.row_ptr)
    assert torch.equal(again.col_idx[:n], ref.col_idx[:n])
    assert torch.equal(again.values[:n], ref.values[:n])
    assert torch.equal(again.block_mass, ref.block_mass)


def test_calib_gram_timeout_then_clean_call():
    ws = synth.Workload("stall_cal", (300,), B=64, h_s=32, h_r=16, h_kv=1, d=8, dtype="bf16",
                        tau=0.9, n_heavy=16, reading=3)
    wr = ws.with_(h_s=16)
    X = sdev.fill_maps(sdev.alloc_maps(ws), ws, 0)
    Y = sdev.fill_maps(sdev.alloc_maps(wr), wr, 1)
    offs = list(zip(X.offsets, Y.offsets))
    assert mf.mf_calib_path(X.maps, Y.maps, offs, ws.lens, 32, 16, 64) == 1

    def call():
        return mf.mf_calib_gram(X.maps, Y.maps, offs, ws.lens, 32, 16, 64)

    ref = call()
    _clean()
    rc, bits = _stalled(call)
    assert rc == mf.MF_ERR_TIMEOUT and bits & 4, (rc, bits)
    again = call()
    _clean()
    assert torch.equal(again, ref)
