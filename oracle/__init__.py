"""CPU oracle for MapFlow's compression and fused retrieval (test infrastructure only).

Plain, slow, float64.  The arithmetic lives in `oracle/oracle.c` (plain loops, one
thread); this module only marshals numpy/torch arrays into it and walks sequences,
query blocks and chunks in the obvious order.  Only the tests, the package smoke check
and the benchmark's CPU-baseline leg use it.  It imports nothing from the CUDA
package, and the CUDA package imports nothing from here.

Every function here is pinned by `tests/test_oracle_pins.py` against brute force,
closed forms, a hand-worked example and textbook causal attention (see that file).
"""
import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

BOUNDARY_EPS = 1e-5


def build(force=False):
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC):
        return _LIB_PATH
    subprocess.run(["gcc", "-O2", "-std=c99", "-shared", "-fPIC", "-o", _LIB_PATH, _SRC, "-lm"],
                   check=True)
    return _LIB_PATH


class _VRef(ctypes.Structure):
    _fields_ = [("V", ctypes.c_void_p), ("dtype", ctypes.c_int), ("paged", ctypes.c_int),
                ("page_size", ctypes.c_int), ("block_table", ctypes.c_void_p),
                ("k_start", ctypes.c_int64), ("h_kv", ctypes.c_int), ("d", ctypes.c_int)]


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.mfo_row_masses.argtypes = [P, I, I, I, I64, I64, I, I, P]
        lib.mfo_row_masses.restype = None
        lib.mfo_select.argtypes = [P, I, D, P, P]
        lib.mfo_select.restype = I
        lib.mfo_gather_block.argtypes = [P, I, I, I, I64, I64, I, I, I, P]
        lib.mfo_gather_block.restype = None
        lib.mfo_retrieve_block.argtypes = [P, I, P, I, I, I, I, P, I, ctypes.POINTER(_VRef), I, I, P]
        lib.mfo_retrieve_block.restype = None
        lib.mfo_calib_gram.argtypes = [P, P, I, I, I, I, I64, P]
        lib.mfo_calib_gram.restype = None
        lib.mfo_calib_solve.argtypes = [P, I, I, D, P, P]
        lib.mfo_calib_solve.restype = I
        lib.mfo_qk_maps.argtypes = [P, P, I, I, I, I, I, I64, D, P]
        lib.mfo_qk_maps.restype = None
        lib.mfo_qk_rows.argtypes = [P, P, I, I, I, I, I, I, I, I64, D, P]
        lib.mfo_qk_rows.restype = None
        _lib = lib
    return _lib


# ----------------------------------------------------------------------------- dtypes

def as_raw(t):
    """(numpy array of the raw elements, dtype code): float32 -> (f32, 0), bf16 -> (uint16, 1),
    float64 -> (f64, 2)."""
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16), 1
        if t.dtype == torch.float32:
            return t.numpy(), 0
        if t.dtype == torch.float64:
            return t.numpy(), 2
        raise TypeError(t.dtype)
    a = np.ascontiguousarray(t)
    if a.dtype == np.uint16:
        return a, 1
    if a.dtype == np.float32:
        return a, 0
    if a.dtype == np.float64:
        return a, 2
    raise TypeError(a.dtype)


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


# ----------------------------------------------------------------------------- compression

def row_masses(slab, L, B, qb):
    """Head-summed block masses mass[0..qb] (float64) of query block qb.
    slab: [h_s, B, >= (qb+1)*B] holding rows qb*B .. qb*B+B-1 of every head."""
    a, code = as_raw(slab)
    h_s, rows, width = a.shape
    assert rows == B and width >= (qb + 1) * B
    out = np.zeros(qb + 1, dtype=np.float64)
    _load().mfo_row_masses(_ptr(a), code, h_s, B, rows * width, width, qb, L, _ptr(out))
    return out


def select(mass, qb, tau):
    """Kept key blocks (ascending int32) of one row and the walk info
    (total, S after the last kept block, S before it, last kept mass, first dropped mass)."""
    m = np.ascontiguousarray(mass, dtype=np.float64)
    kept = np.zeros(qb + 1, dtype=np.int32)
    info = np.zeros(5, dtype=np.float64)
    n = _load().mfo_select(_ptr(m), qb, float(tau), _ptr(kept), _ptr(info))
    return kept[:n].copy(), info


def is_boundary(info, tau, eps=BOUNDARY_EPS):
    """Near-tie rows, where float rounding may legitimately change the kept set: the final
    or pre-final running fraction within eps of tau, or the last kept and first dropped
    masses within eps * total of each other."""
    total, S, S_prev, m_last, m_next = info
    if total <= 0:
        return True
    if abs(S / total - tau) < eps:
        return True
    if S_prev >= 0 and abs(S_prev / total - tau) < eps:
        return True
    if m_last >= 0 and m_next >= 0 and abs(m_last - m_next) < eps * total:
        return True
    return False


def gather_block(slab, L, B, qb, kb):
    a, code = as_raw(slab)
    h_s, rows, width = a.shape
    out = np.zeros((h_s, B, B), dtype=a.dtype)
    _load().mfo_gather_block(_ptr(a), code, h_s, B, rows * width, width, qb, kb, L, _ptr(out))
    return out


def compress_seq(maps, L, B, tau, rows=None):
    """Compress one sequence's dense maps [h_s, Lp, Lp].  Returns a dict with, per query
    block (all of them, or those listed in `rows`): masses, kept blocks, walk info and the
    kept blocks' values [n, h_s, B, B] (raw dtype)."""
    a, code = as_raw(maps)
    nqb = -(-L // B)
    out = {"masses": {}, "kept": {}, "info": {}, "values": {}}
    for qb in (range(nqb) if rows is None else rows):
        slab = a[:, qb * B:(qb + 1) * B, :]
        m = row_masses(slab, L, B, qb)
        kept, info = select(m, qb, tau)
        vals = np.stack([gather_block(slab, L, B, qb, int(kb)) for kb in kept])
        out["masses"][qb], out["kept"][qb], out["info"][qb], out["values"][qb] = m, kept, info, vals
    return out


def compress_pack(maps_per_seq, lens, B, tau):
    """Varlen pack: BSR of all sequences, rows ordered (sequence, query block)."""
    row_ptr, col_idx, values, seq_results = [0], [], [], []
    for maps, L in zip(maps_per_seq, lens):
        r = compress_seq(maps, L, B, tau)
        seq_results.append(r)
        for qb in range(-(-L // B)):
            kept = r["kept"][qb]
            col_idx.extend(kept.tolist())
            values.append(r["values"][qb])
            row_ptr.append(row_ptr[-1] + len(kept))
    return (np.array(row_ptr, dtype=np.int32), np.array(col_idx, dtype=np.int32),
            np.concatenate(values, axis=0), seq_results)


# ----------------------------------------------------------------------------- retrieval

def retrieve_block(vals, kept, qb, B, W_l, V, h_kv, rows, k_start=0, block_table=None,
                   page_size=0):
    """O rows (block-local `rows` = [i0, i1)) of query block qb for one receiver layer, float64
    [i1 - i0, h_r, d].  vals: [n, h_s, B, B] raw; W_l: [h_r, h_s] float32; V: contiguous
    [T, h_kv, d] or paged [pages, page_size, h_kv, d]."""
    va, vcode = as_raw(vals)
    n, h_s = va.shape[0], va.shape[1]
    Va, Vcode = as_raw(V)
    W = np.ascontiguousarray(W_l, dtype=np.float32)
    h_r = W.shape[0]
    d = Va.shape[-1]
    kb = np.ascontiguousarray(kept, dtype=np.int32)
    bt = None
    if block_table is not None:
        bt = np.ascontiguousarray(block_table, dtype=np.int32)
    ref = _VRef(Va.ctypes.data, Vcode, 1 if bt is not None else 0, page_size,
                bt.ctypes.data if bt is not None else None, k_start, h_kv, d)
    i0, i1 = rows
    O = np.zeros((i1 - i0, h_r, d), dtype=np.float64)
    _load().mfo_retrieve_block(_ptr(va), vcode, _ptr(kb), n, qb, B, h_s, _ptr(W), h_r,
                               ctypes.byref(ref), i0, i1, _ptr(O))
    return O


def retrieve_step(bsr_rows, B, W_l, V, h_kv, step, qblock_base, k_starts=None,
                  block_table=None, page_size=0):
    """One chunked-prefill step for one receiver layer.
    bsr_rows(row) -> (kept, vals) gives a BSR row; step = [(q_len, k_len)] per sequence; the
    queries of sequence s are the last q_len tokens of its k_len prefix.  Returns the packed
    O [sum q_len, h_r, d] float64."""
    outs = []
    for s, (q_len, k_len) in enumerate(step):
        if q_len == 0:
            continue
        q0 = k_len - q_len
        O = []
        for qb in range(q0 // B, -(-k_len // B)):
            lo = max(q0, qb * B) - qb * B
            hi = min(k_len, (qb + 1) * B) - qb * B
            kept, vals = bsr_rows(qblock_base[s] + qb)
            bt = block_table[s] if block_table is not None else None
            ks = k_starts[s] if k_starts is not None else 0
            O.append(retrieve_block(vals, kept, qb, B, W_l, V, h_kv, (lo, hi), ks, bt, page_size))
        outs.append(np.concatenate(O, axis=0))
    return np.concatenate(outs, axis=0)


# ----------------------------------------------------------------------------- maps from Q, K

def qk_maps(Q, K, L, B, scale):
    """The sender's causal attention maps of one sequence from its queries Q [L, h_s, d] and
    keys K [L, h_kv, d] (float32 or bfloat16, read exactly): float64 [h_s, Lp, Lp] (Lp = L
    rounded up to B), zero outside j <= i < L.  Query head s reads key head s * h_kv // h_s."""
    qa, qc = as_raw(Q)
    ka, kc = as_raw(K)
    assert qc == kc and qa.shape[0] >= L and ka.shape[0] >= L and qa.shape[2] == ka.shape[2]
    h_s, h_kv, d = qa.shape[1], ka.shape[1], qa.shape[2]
    assert h_s % h_kv == 0
    Lp = -(-L // B) * B
    A = np.empty((h_s, Lp, Lp), dtype=np.float64)
    _load().mfo_qk_maps(_ptr(qa), _ptr(ka), qc, L, h_s, h_kv, d, Lp, float(scale), _ptr(A))
    return A


def qk_slab(Q, K, L, B, qb, scale):
    """Rows of query block qb of the maps of qk_maps: float64 [h_s, B, (qb + 1) * B]."""
    qa, qc = as_raw(Q)
    ka, kc = as_raw(K)
    assert qc == kc
    h_s, h_kv, d = qa.shape[1], ka.shape[1], qa.shape[2]
    width = (qb + 1) * B
    out = np.empty((h_s, B, width), dtype=np.float64)
    _load().mfo_qk_rows(_ptr(qa), _ptr(ka), qc, L, h_s, h_kv, d, qb * B, (qb + 1) * B, width,
                        float(scale), _ptr(out))
    return out


def compress_qk_row(Q, K, L, B, qb, tau, scale):
    """One query block of compression from Q, K: (masses, kept, walk info, values float64)."""
    slab = qk_slab(Q, K, L, B, qb, scale)
    m = row_masses(slab, L, B, qb)
    kept, info = select(m, qb, tau)
    vals = np.stack([gather_block(slab, L, B, qb, int(kb)) for kb in kept])
    return m, kept, info, vals


def compress_qk_seq(Q, K, L, B, tau, scale, rows=None):
    """Compression of one sequence straight from its queries and keys: the maps of qk_maps,
    then the block statistics, selection and kept-block values of compress_seq (values
    float64)."""
    return compress_seq(qk_maps(Q, K, L, B, scale), L, B, tau, rows)


# ----------------------------------------------------------------------------- calibration

def calib_gram(X, Y, L, gram=None):
    """Gram [F, F] (float64, F = h_s + h_r) of the stacked sender / receiver maps of one
    sequence over its causal positions (i < L, j <= i), added to `gram` when given.
    X: [h_s, Lp, Lp], Y: [h_r, Lp, Lp], same dtype (float32 or bfloat16)."""
    xa, xc = as_raw(X)
    ya, yc = as_raw(Y)
    assert xc == yc and xa.shape[1:] == ya.shape[1:]
    h_s, h_r, Lp = xa.shape[0], ya.shape[0], xa.shape[1]
    F = h_s + h_r
    g = np.zeros((F, F), dtype=np.float64) if gram is None else gram
    assert g.shape == (F, F) and g.dtype == np.float64 and g.flags["C_CONTIGUOUS"]
    _load().mfo_calib_gram(_ptr(xa), _ptr(ya), xc, h_s, h_r, L, Lp, _ptr(g))
    return g


def calib_solve(gram, h_s, h_r, ridge=0.0):
    """Least-squares head map from a Gram: W [h_r, h_s] float64 and the residual sum of
    squares per receiver head; raises ValueError when the sender Gram (+ ridge) is not
    positive definite."""
    g = np.ascontiguousarray(gram, dtype=np.float64)
    W = np.zeros((h_r, h_s), dtype=np.float64)
    res = np.zeros(h_r, dtype=np.float64)
    if _load().mfo_calib_solve(_ptr(g), h_s, h_r, float(ridge), _ptr(W), _ptr(res)) != 0:
        raise ValueError("sender Gram is not positive definite")
    return W, res
