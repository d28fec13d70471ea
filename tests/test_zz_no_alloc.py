"""mf_compress_static: compression for callers that cannot allocate device memory.

Such a caller (for example a plugin inside a host program that owns every byte of
device memory through its own pool) passes only inputs and outputs; the scratch comes
from the library's static device array.  The results must be the ones mf_compress
gives with a caller workspace, call after call: the array keeps the previous call's
contents, so two different compressions run back to back through the C ABI and each
is compared with mf_compress.  Compression is exact, so the comparison is bitwise.
This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import synth
from synth import device as sdev


def _compress_both(mf, w):
    pack = sdev.fill_maps(sdev.alloc_maps(w), w, 0)
    rows, cap = sum(w.nqb), w.causal_blocks
    ref = mf.alloc_bsr(rows, cap, w.h_s, w.B, pack.maps.dtype, "cuda", n_causal=w.causal_blocks)
    mf.mf_compress(pack.maps, pack.map_seq_offset, pack.cu_seqlens, max(w.lens), w.h_s, w.B,
                   w.tau, ref)
    out = mf.alloc_bsr(rows, cap, w.h_s, w.B, pack.maps.dtype, "cuda", n_causal=w.causal_blocks)
    # through the C ABI directly: the static variant takes no workspace argument
    d = mf._compress_desc(pack.maps, pack.map_seq_offset, pack.cu_seqlens, max(w.lens), w.h_s,
                          w.B, w.tau, out)
    rc = mf._lib.mf_compress_static(ctypes.byref(d), torch.cuda.current_stream().cuda_stream)
    assert rc == mf.MF_OK, mf._lib.mf_last_error()
    return ref, out


@pytest.mark.gpu
def test_compress_static_equals_compress_two_calls_in_a_row():
    import cross_model_attention_mf_b200 as mf

    cases = [
        synth.Workload("static_a", (300, 129, 64), B=64, h_s=32, h_r=32, h_kv=8, d=128,
                       dtype="bf16", tau=0.95, n_heavy=16, reading=3),
        synth.Workload("static_b", (400, 1), B=128, h_s=16, h_r=8, h_kv=2, d=128, dtype="bf16",
                       tau=0.8, n_heavy=8, reading=1),
    ]
    for w in cases:
        ref, out = _compress_both(mf, w)
        rc, bits = mf.mf_get_status()
        assert rc == mf.MF_OK and bits == 0, (w.name, rc, bits)
        n = int(ref.nnz.cpu()[0])
        assert int(out.nnz.cpu()[0]) == n
        assert torch.equal(out.row_ptr, ref.row_ptr)
        assert torch.equal(out.col_idx[:n], ref.col_idx[:n])
        assert torch.equal(out.values[:n], ref.values[:n])
        assert torch.equal(out.block_mass, ref.block_mass)

    # a descriptor that needs more scratch than the static array is refused up front
    w = cases[0]
    big = mf.CompressDesc()
    big.maps = big.map_seq_offset = big.cu_seqlens = big.row_ptr = big.col_idx = 4096
    big.values = big.nnz_out = 4096
    big.dtype, big.nseq, big.max_seqlen, big.h_s, big.B, big.tau = 1, 64, 262144, 4, 64, 0.9
    big.capacity_blocks = 1
    assert mf._lib.mf_compress_static(ctypes.byref(big), None) == mf.MF_ERR_UNSUPPORTED
    assert b"static" in mf._lib.mf_last_error()
