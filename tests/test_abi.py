"""The C ABI library (no GPU needed): it loads, exports every function include/mf.h
declares, mirrors its structs, and rejects bad descriptors on the host before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def mf():
    import __graft_entry__
    __graft_entry__.load_builder().build()
    import cross_model_attention_mf_b200 as mf
    return mf


def header_functions():
    txt = open(os.path.join(ROOT, "include", "mf.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(mf_[a-z_]+)\s*\(", txt)))


def test_exports_every_declared_function(mf):
    lib = ctypes.CDLL(mf.LIB_PATH)
    names = header_functions()
    assert {"mf_compress", "mf_map_retrieve", "mf_compress_workspace_size", "mf_get_status"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_struct_mirrors(mf):
    assert mf._lib.mf_abi_struct_size(0) == ctypes.sizeof(mf.CompressDesc)
    assert mf._lib.mf_abi_struct_size(1) == ctypes.sizeof(mf.BsrDesc)
    assert mf._lib.mf_abi_struct_size(2) == ctypes.sizeof(mf.RetrieveDesc)
    assert mf._lib.mf_abi_struct_size(7) == 0
    assert "sm_100a" in mf.mf_version()


def test_workspace_size_bounds(mf):
    small = mf.mf_compress_workspace_size(1, 256, 32, 10)
    big = mf.mf_compress_workspace_size(16, 8192, 64, 100000)
    assert 0 < small < big
    # per-sequence meta + float64 masses of 128*129/2 blocks per sequence + one 8-byte
    # look-back flag per query block + kept rows
    assert big >= 16 * (128 * 129 // 2) * 8 + 16 * 128 * 8 + 100000 * 4
    assert mf.mf_compress_workspace_size(1, 100, 64, 0) % 256 == 0


def _compress_desc(mf, **kw):
    d = mf.CompressDesc()
    d.maps = d.map_seq_offset = d.cu_seqlens = d.row_ptr = d.col_idx = d.values = d.nnz_out = 4096
    d.dtype, d.nseq, d.max_seqlen, d.h_s, d.B, d.tau, d.capacity_blocks = 1, 1, 128, 4, 64, 0.9, 8
    for k, v in kw.items():
        setattr(d, k, v)
    return d


@pytest.mark.parametrize("field,value", [("B", 48), ("tau", 1.5), ("tau", -0.1), ("h_s", 0),
                                         ("nseq", 0), ("dtype", 5), ("maps", 0),
                                         ("capacity_blocks", -1), ("values", 4100)])
def test_compress_rejects_bad_descriptor(mf, field, value):
    d = _compress_desc(mf, **{field: value})
    rc = mf._lib.mf_compress(ctypes.byref(d), ctypes.c_void_p(4096), 1 << 30, None)
    assert rc == mf.MF_ERR_INVALID
    assert mf._lib.mf_last_error().decode()


def test_compress_rejects_small_workspace(mf):
    d = _compress_desc(mf)
    rc = mf._lib.mf_compress(ctypes.byref(d), ctypes.c_void_p(4096), 16, None)
    assert rc == mf.MF_ERR_INVALID and b"workspace" in mf._lib.mf_last_error()
    rc = mf._lib.mf_compress(ctypes.byref(d), ctypes.c_void_p(4096 + 8), 1 << 30, None)
    assert rc == mf.MF_ERR_INVALID and b"aligned" in mf._lib.mf_last_error()


def test_compress_rejects_too_many_blocks(mf):
    d = _compress_desc(mf, max_seqlen=4097 * 64)
    rc = mf._lib.mf_compress(ctypes.byref(d), ctypes.c_void_p(4096), 1 << 40, None)
    assert rc == mf.MF_ERR_UNSUPPORTED


def _retrieve_desc(mf, bsr_arr, lm, **kw):
    d = mf.RetrieveDesc()
    d.layers = bsr_arr
    d.n_sender_layers = 1
    d.map_dtype = d.v_dtype = 1
    d.h_s, d.B = 32, 64
    d.layer_map = ctypes.cast(lm, ctypes.c_void_p)
    d.l_r_begin, d.l_r_end = 0, 1
    d.W = d.V = d.O = d.cu_seqlens_q = d.cu_seqlens_k = d.qblock_base = 4096
    d.total_k, d.nseq, d.max_seqlen_q = 8192, 1, 8192
    d.h_r, d.h_kv, d.d = 32, 8, 128
    d.total_q = 8192
    for k, v in kw.items():
        setattr(d, k, v)
    return d


def test_retrieve_path_selection(mf):
    arr = (mf.BsrDesc * 1)(mf.BsrDesc(4096, 4096, 4096, 100))
    lm = (ctypes.c_int32 * 1)(0)
    P = mf._lib.mf_retrieve_path
    assert P(ctypes.byref(_retrieve_desc(mf, arr, lm))) == 1                     # Ministral-like
    assert P(ctypes.byref(_retrieve_desc(mf, arr, lm, B=128, h_r=24))) == 1      # long context, gq 3
    assert P(ctypes.byref(_retrieve_desc(mf, arr, lm, h_s=40))) == 1             # Qwen-like
    assert P(ctypes.byref(_retrieve_desc(mf, arr, lm, map_dtype=0, v_dtype=0, B=32, h_s=4,
                                         h_r=2, h_kv=1, d=64))) == 0             # tiny float32
    assert P(ctypes.byref(_retrieve_desc(mf, arr, lm, flags=mf.MF_RETRIEVE_FORCE_SIMT))) == 0
    assert P(ctypes.byref(_retrieve_desc(mf, arr, lm, h_r=32, h_kv=4))) == 0      # gq 8: SIMT
    assert P(ctypes.byref(_retrieve_desc(mf, arr, lm, paged=1, page_size=16, n_pages=10,
                                         max_pages=4, block_table=4096))) == 1


@pytest.mark.parametrize("field,value", [("h_r", 30), ("l_r_end", 2), ("d", 0), ("nseq", 0),
                                         ("W", 0), ("map_dtype", 9), ("l_r_begin", -1),
                                         ("flags", 8), ("V", 4104)])
def test_retrieve_rejects_bad_descriptor(mf, field, value):
    arr = (mf.BsrDesc * 1)(mf.BsrDesc(4096, 4096, 4096, 100))
    lm = (ctypes.c_int32 * 2)(0, 3)
    d = _retrieve_desc(mf, arr, lm, **{field: value})
    assert mf._lib.mf_map_retrieve(ctypes.byref(d), None) == mf.MF_ERR_INVALID
    assert mf._lib.mf_retrieve_path(ctypes.byref(d)) == -1


def test_retrieve_rejects_unmapped_layer(mf):
    arr = (mf.BsrDesc * 1)(mf.BsrDesc(4096, 4096, 0, 100))
    lm = (ctypes.c_int32 * 1)(0)
    d = _retrieve_desc(mf, arr, lm)
    assert mf._lib.mf_map_retrieve(ctypes.byref(d), None) == mf.MF_ERR_INVALID


def test_calib_host_validation(mf):
    d = mf.CalibDesc()
    assert mf._lib.mf_calib_gram(None, None, 0, None) == mf.MF_ERR_INVALID
    nb = ctypes.c_size_t(0)
    assert mf._lib.mf_calib_workspace_size(ctypes.byref(d), ctypes.byref(nb)) == mf.MF_ERR_INVALID
    so = (ctypes.c_int64 * 1)(0)
    ro = (ctypes.c_int64 * 1)(3)  # not a multiple of 8 elements
    ln = (ctypes.c_int32 * 1)(100)
    d = mf.CalibDesc(4096, 4096, mf.MF_BF16, ctypes.cast(so, ctypes.c_void_p), ctypes.cast(ro, ctypes.c_void_p),
                     ctypes.cast(ln, ctypes.c_void_p), 1, 32, 32, 64, 4096)
    assert mf._lib.mf_calib_gram(ctypes.byref(d), None, 0, None) == mf.MF_ERR_INVALID
    assert b"multiples of 8" in mf._lib.mf_last_error()
    ro[0] = 0
    d.h_s = 65
    assert mf._lib.mf_calib_path(ctypes.byref(d)) == -1
    d.h_s = 32
    assert mf._lib.mf_calib_path(ctypes.byref(d)) == 1
    d.h_s = 12
    assert mf._lib.mf_calib_path(ctypes.byref(d)) == 0
    d.h_s, d.h_r, d.dtype = 40, 40, mf.MF_F32  # F = 80 needs the tensor-core path
    assert mf._lib.mf_calib_gram(ctypes.byref(d), None, 0, None) == mf.MF_ERR_UNSUPPORTED
    assert mf._lib.mf_calib_solve(None, 4, 4, 0.0, None, None, None) == mf.MF_ERR_INVALID
    assert mf._lib.mf_calib_solve(4096, 4, 4, -1.0, 4096, None, None) == mf.MF_ERR_INVALID
    assert mf._lib.mf_calib_solve(4096, 65, 4, 0.0, 4096, None, None) == mf.MF_ERR_UNSUPPORTED


def test_retrieve_multi_fusing_rules(mf):
    """Receivers of one sender share launches only when they share its blocks and the packing."""
    arr = (mf.BsrDesc * 1)(mf.BsrDesc(4096, 4096, 4096, 100))
    other = (mf.BsrDesc * 1)(mf.BsrDesc(4096, 8192, 4096, 100))
    lm = (ctypes.c_int32 * 1)(0)
    F = mf._lib.mf_retrieve_multi_fused

    def many(*ds):
        a = (mf.RetrieveDesc * len(ds))()
        for k, d in enumerate(ds):
            a[k] = d
        return a

    base = _retrieve_desc(mf, arr, lm)
    small = _retrieve_desc(mf, arr, lm, h_r=8, h_kv=2, W=8192, V=8192, O=16384)  # another receiver
    assert F(many(base, small), 2) == 1
    assert F(many(base, small, small, base, small), 5) == 1          # two launches per step
    assert F(many(base, _retrieve_desc(mf, other, lm)), 2) == 0       # other sender blocks
    assert F(many(base, _retrieve_desc(mf, arr, lm, cu_seqlens_q=12288)), 2) == 0  # other packing
    assert F(many(base, _retrieve_desc(mf, arr, lm, h_r=32, h_kv=4)), 2) == 0      # SIMT receiver
    assert F(many(base, _retrieve_desc(mf, arr, lm, h_r=30)), 2) == -1             # invalid
    assert mf._lib.mf_map_retrieve_multi(many(base), 0, None) == mf.MF_ERR_INVALID
    assert mf._lib.mf_map_retrieve_multi(many(base, _retrieve_desc(mf, arr, lm, d=0)), 2,
                                         None) == mf.MF_ERR_INVALID


def test_compress_qk_descriptor_and_validation(mf):
    """The binding fills every field of mf_compress_qk_desc; the host checks reject what the
    kernels do not take, before any launch."""
    import torch
    Q = torch.zeros(100, 8, 128, dtype=torch.bfloat16)
    K = torch.zeros(100, 2, 128, dtype=torch.bfloat16)
    cu = torch.tensor([0, 60, 100], dtype=torch.int32)
    out = mf.alloc_bsr(2, 4, 8, 64, torch.bfloat16, "cpu", n_causal=4)
    d = mf._compress_qk_desc(Q, K, cu, 60, 64, 0.9, out)
    assert (d.Q, d.K, d.cu_seqlens) == (Q.data_ptr(), K.data_ptr(), cu.data_ptr())
    assert (d.nseq, d.max_seqlen, d.T, d.h_s, d.h_kv, d.d, d.B) == (2, 60, 100, 8, 2, 128, 64)
    assert d.dtype == mf.MF_BF16 and d.capacity_blocks == 4 and d.block_mass_out == out.block_mass.data_ptr()
    n = ctypes.c_size_t(0)
    assert mf._lib.mf_compress_qk_workspace_size(ctypes.byref(d), ctypes.byref(n)) == mf.MF_OK
    assert n.value >= 8 * 2 * 64 * 8  # (m, l) of every (head, causal block, row)
    for field, value, rc in [("d", 64, mf.MF_ERR_UNSUPPORTED), ("B", 32, mf.MF_ERR_UNSUPPORTED),
                             ("dtype", mf.MF_F32, mf.MF_ERR_UNSUPPORTED), ("h_kv", 3, mf.MF_ERR_INVALID),
                             ("tau", 1.5, mf.MF_ERR_INVALID), ("nseq", 0, mf.MF_ERR_INVALID),
                             ("scale", -1.0, mf.MF_ERR_INVALID)]:
        bad = mf._compress_qk_desc(Q, K, cu, 60, 64, 0.9, out)
        setattr(bad, field, value)
        assert mf._lib.mf_compress_qk(ctypes.byref(bad), ctypes.c_void_p(4096), 1 << 30, None) == rc, field
    assert mf._lib.mf_abi_struct_size(4) == ctypes.sizeof(mf.CompressQkDesc)


def test_multi_receiver_binding_descriptors(mf):
    """The binding's several-receiver descriptors carry each receiver's own W, V, O, heads and
    paging, and the shared packing; the host fusing decision follows from them (no launch)."""
    import torch
    layers = [mf.BSR(torch.zeros(3, dtype=torch.int32), torch.zeros(4, dtype=torch.int32),
                     torch.zeros(4, 8, 64, 64, dtype=torch.bfloat16), torch.zeros(1, dtype=torch.int32))]
    cu = torch.tensor([0, 100], dtype=torch.int32)
    qb = torch.zeros(1, dtype=torch.int32)
    rs = [mf.Receiver([0], torch.zeros(1, 8, 8), torch.zeros(1, 100, 2, 128, dtype=torch.bfloat16), 8, 2,
                      O=torch.zeros(1, 100, 8, 128, dtype=torch.bfloat16)),
          mf.Receiver([0], torch.zeros(1, 4, 8), torch.zeros(1, 100, 1, 128, dtype=torch.bfloat16), 4, 1,
                      O=torch.zeros(1, 100, 4, 128, dtype=torch.bfloat16))]
    arr, keep, outs = mf._multi_descs(layers, rs, cu, cu, qb, 100, 100, None)
    assert [d.h_r for d in arr] == [8, 4] and [d.h_kv for d in arr] == [2, 1]
    assert arr[0].W == rs[0].W.data_ptr() and arr[1].V == rs[1].V.data_ptr()
    assert arr[0].O == outs[0].data_ptr() and arr[1].O == outs[1].data_ptr()
    assert arr[0].cu_seqlens_q == arr[1].cu_seqlens_q == cu.data_ptr()
    assert mf._lib.mf_retrieve_multi_fused(arr, 2) == 1
    # a receiver whose GQA group exceeds 4 heads takes the SIMT kernel: no shared launch
    rs.append(mf.Receiver([0], torch.zeros(1, 16, 8), torch.zeros(1, 100, 2, 128, dtype=torch.bfloat16),
                          16, 2, O=torch.zeros(1, 100, 16, 128, dtype=torch.bfloat16)))
    arr, keep, outs = mf._multi_descs(layers, rs, cu, cu, qb, 100, 100, None)
    assert mf._lib.mf_retrieve_multi_fused(arr, 3) == 0


def test_wait_limit_setter(mf):
    """The bounded-wait limit is host state read at each launch: setting and restoring it needs
    no device (the GPU tests in test_gpu_timeout.py make a wait run out with it)."""
    assert mf._lib.mf_set_wait_limit(5_000_000, 1) == mf.MF_OK
    assert mf._lib.mf_set_wait_limit(0, 0) == mf.MF_OK
