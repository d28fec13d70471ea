"""Python binding of libmf (include/mf.h): MapFlow compression and fused retrieval on B200.

Argument marshalling only: every step of the path runs in the CUDA kernels of
libmf.so.  PyTorch supplies device memory and the current stream.  Importing
this package fails loudly when libmf.so is missing; there is no fallback.

Functions mirror the C entry points:
    mf_compress(...)        -> BSR (row_ptr, col_idx, values, nnz)
    mf_compress_qk(...)     -> BSR, straight from the sender's Q and K (no dense map)
    mf_map_retrieve(...)    -> O
    mf_map_retrieve_multi(...) -> [O]   (one sender, several receivers)
    mf_prefix_hashes(...), BlockCache(...).put / get / stats   (prefix-hash block cache)
    mf_get_status()         -> (status, bits)
    mf_set_wait_limit(...)  bounded-wait limit (and a test stall) of the tensor-core kernels
    mf_compress_workspace_size(...), mf_retrieve_path(...), mf_version()
    mf_calib_gram(...), mf_calib_solve(...), mf_calib_path(...)   (head-map calibration)
"""
import ctypes
import os
from dataclasses import dataclass
from typing import List, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# MF_LIBRARY may point at another build of the same ABI (for example a traced one)
LIB_PATH = os.environ.get("MF_LIBRARY") or os.path.join(_HERE, "libmf.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m cross_model_attention_mf_b200.build` "
                      "(nvcc, sm_100a); this package has no CPU or library fallback")

_lib = ctypes.CDLL(LIB_PATH)

MF_OK, MF_ERR_INVALID, MF_ERR_UNSUPPORTED, MF_ERR_CAPACITY, MF_ERR_CUDA, MF_ERR_TIMEOUT, \
    MF_ERR_DEVICE_INDEX = range(7)
MF_F32, MF_BF16 = 0, 1
MF_RETRIEVE_FORCE_SIMT = 1
MF_RETRIEVE_O_F32 = 2
MF_RETRIEVE_P_SPLIT = 4

_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64


class CompressDesc(ctypes.Structure):
    _fields_ = [("maps", _P), ("dtype", ctypes.c_int), ("map_seq_offset", _P), ("cu_seqlens", _P),
                ("nseq", _I32), ("max_seqlen", _I32), ("h_s", _I32), ("B", _I32),
                ("tau", ctypes.c_double), ("row_ptr", _P), ("col_idx", _P), ("values", _P),
                ("capacity_blocks", _I64), ("nnz_out", _P), ("block_mass_out", _P)]


class CompressQkDesc(ctypes.Structure):
    _fields_ = [("Q", _P), ("K", _P), ("dtype", ctypes.c_int), ("cu_seqlens", _P),
                ("nseq", _I32), ("max_seqlen", _I32), ("T", _I64), ("h_s", _I32), ("h_kv", _I32),
                ("d", _I32), ("scale", ctypes.c_float), ("B", _I32), ("tau", ctypes.c_double),
                ("row_ptr", _P), ("col_idx", _P), ("values", _P), ("capacity_blocks", _I64),
                ("nnz_out", _P), ("block_mass_out", _P), ("lse_out", _P)]


class CacheDesc(ctypes.Structure):
    _fields_ = [("pool", _P), ("pool_bytes", ctypes.c_size_t), ("h_s", _I32), ("B", _I32),
                ("dtype", ctypes.c_int)]


class BsrDesc(ctypes.Structure):
    _fields_ = [("row_ptr", _P), ("col_idx", _P), ("values", _P), ("capacity_blocks", _I64)]


class RetrieveDesc(ctypes.Structure):
    _fields_ = [("layers", ctypes.POINTER(BsrDesc)), ("n_sender_layers", _I32),
                ("map_dtype", ctypes.c_int), ("h_s", _I32), ("B", _I32), ("layer_map", _P),
                ("l_r_begin", _I32), ("l_r_end", _I32), ("W", _P), ("V", _P),
                ("v_dtype", ctypes.c_int), ("v_layer_stride", _I64), ("paged", _I32),
                ("page_size", _I32), ("n_pages", _I32), ("max_pages", _I32), ("block_table", _P),
                ("total_k", _I64), ("cu_seqlens_q", _P), ("cu_seqlens_k", _P),
                ("qblock_base", _P), ("nseq", _I32), ("max_seqlen_q", _I32), ("h_r", _I32),
                ("h_kv", _I32), ("d", _I32), ("O", _P), ("o_layer_stride", _I64),
                ("total_q", _I32), ("flags", _I32)]


class CalibDesc(ctypes.Structure):
    _fields_ = [("sender_maps", _P), ("receiver_maps", _P), ("dtype", ctypes.c_int),
                ("sender_seq_offset", _P), ("receiver_seq_offset", _P), ("seqlens", _P),
                ("nseq", _I32), ("h_s", _I32), ("h_r", _I32), ("B", _I32), ("gram", _P)]


_lib.mf_compress_workspace_size.argtypes = [ctypes.POINTER(CompressDesc), ctypes.POINTER(ctypes.c_size_t)]
_lib.mf_compress_workspace_size.restype = ctypes.c_int
_lib.mf_compress.argtypes = [ctypes.POINTER(CompressDesc), _P, ctypes.c_size_t, _P]
_lib.mf_compress.restype = ctypes.c_int
_lib.mf_compress_static.argtypes = [ctypes.POINTER(CompressDesc), _P]
_lib.mf_compress_static.restype = ctypes.c_int
_lib.mf_compress_qk_workspace_size.argtypes = [ctypes.POINTER(CompressQkDesc), ctypes.POINTER(ctypes.c_size_t)]
_lib.mf_compress_qk_workspace_size.restype = ctypes.c_int
_lib.mf_compress_qk.argtypes = [ctypes.POINTER(CompressQkDesc), _P, ctypes.c_size_t, _P]
_lib.mf_compress_qk.restype = ctypes.c_int
_lib.mf_prefix_hashes.argtypes = [_P, _I64, _I32, _P]
_lib.mf_prefix_hashes.restype = ctypes.c_int
_lib.mf_cache_create.argtypes = [ctypes.POINTER(CacheDesc), ctypes.POINTER(_P)]
_lib.mf_cache_create.restype = ctypes.c_int
_lib.mf_cache_destroy.argtypes = [_P]
_lib.mf_cache_destroy.restype = None
_lib.mf_cache_put.argtypes = [_P, _I32, ctypes.POINTER(BsrDesc), _P, _P, _I64, _I32, _P,
                              ctypes.POINTER(_I64), _P]
_lib.mf_cache_put.restype = ctypes.c_int
_lib.mf_cache_get.argtypes = [_P, _I32, _P, _I32, _P, _P, _P, _I64, ctypes.POINTER(_I32), _P]
_lib.mf_cache_get.restype = ctypes.c_int
_lib.mf_cache_stats.argtypes = [_P, _P]
_lib.mf_cache_stats.restype = ctypes.c_int
_lib.mf_map_retrieve.argtypes = [ctypes.POINTER(RetrieveDesc), _P]
_lib.mf_map_retrieve.restype = ctypes.c_int
_lib.mf_map_retrieve_multi.argtypes = [ctypes.POINTER(RetrieveDesc), ctypes.c_int, _P]
_lib.mf_map_retrieve_multi.restype = ctypes.c_int
_lib.mf_retrieve_multi_fused.argtypes = [ctypes.POINTER(RetrieveDesc), ctypes.c_int]
_lib.mf_retrieve_multi_fused.restype = ctypes.c_int
_lib.mf_retrieve_path.argtypes = [ctypes.POINTER(RetrieveDesc)]
_lib.mf_retrieve_path.restype = ctypes.c_int
_lib.mf_set_wait_limit.argtypes = [ctypes.c_uint64, ctypes.c_int]
_lib.mf_set_wait_limit.restype = ctypes.c_int
_lib.mf_get_status.argtypes = [_P, ctypes.POINTER(ctypes.c_uint32)]
_lib.mf_get_status.restype = ctypes.c_int
_lib.mf_last_error.argtypes = []
_lib.mf_last_error.restype = ctypes.c_char_p
_lib.mf_version.argtypes = []
_lib.mf_version.restype = ctypes.c_char_p
_lib.mf_abi_struct_size.argtypes = [ctypes.c_int]
_lib.mf_abi_struct_size.restype = ctypes.c_size_t
_lib.mf_calib_workspace_size.argtypes = [ctypes.POINTER(CalibDesc), ctypes.POINTER(ctypes.c_size_t)]
_lib.mf_calib_workspace_size.restype = ctypes.c_int
_lib.mf_calib_gram.argtypes = [ctypes.POINTER(CalibDesc), _P, ctypes.c_size_t, _P]
_lib.mf_calib_gram.restype = ctypes.c_int
_lib.mf_calib_solve.argtypes = [_P, _I32, _I32, ctypes.c_double, _P, _P, _P]
_lib.mf_calib_solve.restype = ctypes.c_int
_lib.mf_calib_path.argtypes = [ctypes.POINTER(CalibDesc)]
_lib.mf_calib_path.restype = ctypes.c_int

for _k, _s in ((0, CompressDesc), (1, BsrDesc), (2, RetrieveDesc), (3, CalibDesc)):
    if _lib.mf_abi_struct_size(_k) != ctypes.sizeof(_s):
        raise ImportError(f"libmf.so struct {_s.__name__} size mismatch: rebuild the library")


class MFError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"mf status {status}: {msg}")
        self.status = status


def _check(rc):
    if rc != MF_OK:
        raise MFError(rc, _lib.mf_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _dt(t: torch.Tensor):
    if t.dtype == torch.float32:
        return MF_F32
    if t.dtype == torch.bfloat16:
        return MF_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def mf_version() -> str:
    return _lib.mf_version().decode()


@dataclass
class BSR:
    """Compressed sender layer (device tensors)."""
    row_ptr: torch.Tensor   # int32 [R + 1]
    col_idx: torch.Tensor   # int32 [capacity]
    values: torch.Tensor    # [capacity, h_s, B, B]
    nnz: torch.Tensor       # int32 [1]
    block_mass: Optional[torch.Tensor] = None  # float64 [causal blocks]

    @property
    def capacity(self) -> int:
        return self.values.shape[0]

    def desc(self) -> BsrDesc:
        return BsrDesc(self.row_ptr.data_ptr(), self.col_idx.data_ptr(), self.values.data_ptr(),
                       self.capacity)


def _compress_desc(maps, map_seq_offset, cu_seqlens, max_seqlen, h_s, B, tau, out: BSR):
    return CompressDesc(_ptr(maps), _dt(maps), _ptr(map_seq_offset), _ptr(cu_seqlens),
                        cu_seqlens.numel() - 1, int(max_seqlen), int(h_s), int(B), float(tau),
                        _ptr(out.row_ptr), _ptr(out.col_idx), _ptr(out.values), out.capacity,
                        _ptr(out.nnz), _ptr(out.block_mass))


def mf_compress_workspace_size(nseq: int, max_seqlen: int, B: int, capacity: int) -> int:
    d = CompressDesc()
    d.nseq, d.max_seqlen, d.B, d.capacity_blocks = nseq, max_seqlen, B, capacity
    n = ctypes.c_size_t(0)
    _check(_lib.mf_compress_workspace_size(ctypes.byref(d), ctypes.byref(n)))
    return n.value


def alloc_bsr(n_rows: int, capacity: int, h_s: int, B: int, dtype, device, n_causal: int = 0) -> BSR:
    """Output buffers of one compressed layer (PyTorch allocations)."""
    return BSR(torch.empty(n_rows + 1, dtype=torch.int32, device=device),
               torch.empty(max(capacity, 1), dtype=torch.int32, device=device),
               torch.empty((max(capacity, 1), h_s, B, B), dtype=dtype, device=device),
               torch.empty(1, dtype=torch.int32, device=device),
               torch.empty(n_causal, dtype=torch.float64, device=device) if n_causal else None)


def mf_compress(maps: torch.Tensor, map_seq_offset: torch.Tensor, cu_seqlens: torch.Tensor,
                max_seqlen: int, h_s: int, B: int, tau: float, out: BSR,
                workspace: Optional[torch.Tensor] = None, stream=None) -> BSR:
    """Enqueue compression of one sender layer into `out` (see mf.h for the layout)."""
    d = _compress_desc(maps, map_seq_offset, cu_seqlens, max_seqlen, h_s, B, tau, out)
    need = ctypes.c_size_t(0)
    _check(_lib.mf_compress_workspace_size(ctypes.byref(d), ctypes.byref(need)))
    if workspace is None:
        workspace = torch.empty(need.value, dtype=torch.uint8, device=maps.device)
    _check(_lib.mf_compress(ctypes.byref(d), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def _compress_qk_desc(Q, K, cu_seqlens, max_seqlen, B, tau, out: BSR, scale=0.0, lse=None):
    return CompressQkDesc(_ptr(Q), _ptr(K), _dt(Q), _ptr(cu_seqlens), cu_seqlens.numel() - 1,
                          int(max_seqlen), Q.shape[0], Q.shape[1], K.shape[1], Q.shape[2],
                          float(scale), int(B), float(tau), _ptr(out.row_ptr), _ptr(out.col_idx),
                          _ptr(out.values), out.capacity, _ptr(out.nnz), _ptr(out.block_mass),
                          _ptr(lse))


def mf_compress_qk(Q: torch.Tensor, K: torch.Tensor, cu_seqlens: torch.Tensor, max_seqlen: int,
                   B: int, tau: float, out: BSR, scale: float = 0.0,
                   lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                   stream=None) -> BSR:
    """Enqueue compression straight from the sender's Q [T, h_s, d] and K [T, h_kv, d]
    (bfloat16) into `out` (values bfloat16); scale 0 means 1 / sqrt(d); lse (optional float32
    [h_s, T]) receives each row's log2-sum-exp of the scaled scores."""
    d = _compress_qk_desc(Q, K, cu_seqlens, max_seqlen, B, tau, out, scale, lse)
    need = ctypes.c_size_t(0)
    _check(_lib.mf_compress_qk_workspace_size(ctypes.byref(d), ctypes.byref(need)))
    if workspace is None:
        workspace = torch.empty(need.value, dtype=torch.uint8, device=Q.device)
    _check(_lib.mf_compress_qk(ctypes.byref(d), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def mf_compress_qk_workspace_size(nseq: int, max_seqlen: int, T: int, h_s: int, h_kv: int,
                                  capacity: int, B: int = 64, d: int = 128) -> int:
    desc = CompressQkDesc()
    desc.Q = desc.K = desc.cu_seqlens = desc.row_ptr = desc.col_idx = desc.values = desc.nnz_out = 256
    desc.dtype, desc.nseq, desc.max_seqlen, desc.T = MF_BF16, nseq, max_seqlen, T
    desc.h_s, desc.h_kv, desc.d, desc.B, desc.tau, desc.capacity_blocks = h_s, h_kv, d, B, 0.5, capacity
    n = ctypes.c_size_t(0)
    _check(_lib.mf_compress_qk_workspace_size(ctypes.byref(desc), ctypes.byref(n)))
    return n.value


MF_STATIC_WORKSPACE_BYTES = 8 << 20


def mf_compress_static(maps: torch.Tensor, map_seq_offset: torch.Tensor, cu_seqlens: torch.Tensor,
                       max_seqlen: int, h_s: int, B: int, tau: float, out: BSR,
                       stream=None) -> BSR:
    """Same as mf_compress, for callers that cannot allocate device memory: the scratch
    comes from the library's static device array (see mf.h); nothing is allocated here."""
    d = _compress_desc(maps, map_seq_offset, cu_seqlens, max_seqlen, h_s, B, tau, out)
    _check(_lib.mf_compress_static(ctypes.byref(d), _stream(stream)))
    return out


def _retrieve_desc(layers: Sequence[BSR], layer_map: Sequence[int], l_r_range, W, V, O,
                   cu_seqlens_q, cu_seqlens_k, qblock_base, max_seqlen_q, h_s, B, h_r, h_kv,
                   v_layer_stride=0, o_layer_stride=0, paged=None, flags=0):
    arr = (BsrDesc * len(layers))(*[b.desc() for b in layers])
    lm = (ctypes.c_int32 * len(layer_map))(*layer_map)
    d = RetrieveDesc()
    d.layers = arr
    d.n_sender_layers = len(layers)
    d.map_dtype = _dt(layers[0].values)
    d.h_s, d.B = h_s, B
    d.layer_map = ctypes.cast(lm, _P)
    d.l_r_begin, d.l_r_end = l_r_range
    d.W, d.V = _ptr(W), _ptr(V)
    d.v_dtype = _dt(V)
    d.v_layer_stride = v_layer_stride
    if paged is not None:
        block_table, page_size = paged
        d.paged, d.page_size = 1, page_size
        d.n_pages = V.shape[-4]
        d.max_pages = block_table.shape[-1]
        d.block_table = _ptr(block_table)
    else:
        d.total_k = V.shape[-3]
    d.cu_seqlens_q, d.cu_seqlens_k, d.qblock_base = _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), _ptr(qblock_base)
    d.nseq = cu_seqlens_q.numel() - 1
    d.max_seqlen_q = int(max_seqlen_q)
    d.h_r, d.h_kv, d.d = h_r, h_kv, V.shape[-1]
    d.O = _ptr(O)
    d.o_layer_stride = o_layer_stride
    d.total_q = O.shape[-3]
    d.flags = flags
    return d, (arr, lm)  # keep the ctypes arrays alive


def mf_map_retrieve(layers: Sequence[BSR], layer_map: Sequence[int], W: torch.Tensor,
                    V: torch.Tensor, cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor,
                    qblock_base: torch.Tensor, max_seqlen_q: int, h_r: int, h_kv: int,
                    O: Optional[torch.Tensor] = None, l_r_range=None, total_q: Optional[int] = None,
                    paged=None, v_layer_stride: int = 0, force_simt: bool = False,
                    o_f32: bool = False, p_split: bool = False, stream=None) -> torch.Tensor:
    """Enqueue fused retrieval for receiver layers l_r_range (default: all of layer_map).
    O: [n_layers, T_q, h_r, d] (allocated when None; float32 with o_f32, else V's dtype).
    paged = (block_table, page_size).  p_split: P.V takes P as a bf16 pair in every query
    block (MF_RETRIEVE_P_SPLIT)."""
    if l_r_range is None:
        l_r_range = (0, len(layer_map))
    n_l = l_r_range[1] - l_r_range[0]
    h_s, B = layers[0].values.shape[1], layers[0].values.shape[2]
    if O is None:
        if total_q is None:
            raise ValueError("total_q is needed to allocate O")
        O = torch.empty((n_l, total_q, h_r, V.shape[-1]), dtype=torch.float32 if o_f32 else V.dtype,
                        device=V.device)
    flags = ((MF_RETRIEVE_FORCE_SIMT if force_simt else 0) | (MF_RETRIEVE_O_F32 if o_f32 else 0)
             | (MF_RETRIEVE_P_SPLIT if p_split else 0))
    d, keep = _retrieve_desc(layers, layer_map, l_r_range, W, V, O, cu_seqlens_q, cu_seqlens_k,
                             qblock_base, max_seqlen_q, h_s, B, h_r, h_kv, v_layer_stride,
                             0, paged, flags)
    _check(_lib.mf_map_retrieve(ctypes.byref(d), _stream(stream)))
    del keep
    return O


@dataclass
class Receiver:
    """One receiver model of a shared sender: its layer map, head map W [L_r, h_r, h_s],
    V ([L_r, T_k, h_kv, d] or paged [L_r, pages, page, h_kv, d]) and output O."""
    layer_map: Sequence[int]
    W: torch.Tensor
    V: torch.Tensor
    h_r: int
    h_kv: int
    O: Optional[torch.Tensor] = None
    paged: Optional[tuple] = None
    v_layer_stride: int = 0


def _multi_descs(layers, receivers, cu_seqlens_q, cu_seqlens_k, qblock_base, max_seqlen_q,
                 total_q, l_r_range):
    h_s, B = layers[0].values.shape[1], layers[0].values.shape[2]
    arr = (RetrieveDesc * len(receivers))()
    keep, outs = [], []
    for k, r in enumerate(receivers):
        rng = l_r_range if l_r_range is not None else (0, len(r.layer_map))
        O = r.O
        if O is None:
            if total_q is None:
                raise ValueError("total_q is needed to allocate O")
            O = torch.empty((rng[1] - rng[0], total_q, r.h_r, r.V.shape[-1]), dtype=r.V.dtype,
                            device=r.V.device)
        d, kp = _retrieve_desc(layers, r.layer_map, rng, r.W, r.V, O, cu_seqlens_q, cu_seqlens_k,
                               qblock_base, max_seqlen_q, h_s, B, r.h_r, r.h_kv, r.v_layer_stride,
                               0, r.paged, 0)
        arr[k] = d
        keep.append(kp)
        outs.append(O)
    return arr, keep, outs


def mf_map_retrieve_multi(layers: Sequence[BSR], receivers: Sequence[Receiver],
                          cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor,
                          qblock_base: torch.Tensor, max_seqlen_q: int,
                          total_q: Optional[int] = None, l_r_range=None,
                          stream=None) -> List[torch.Tensor]:
    """Retrieval for several receivers of one sender's compressed layers (one O per receiver);
    up to four receivers share each launch when they can (mf_retrieve_multi_fused)."""
    arr, keep, outs = _multi_descs(layers, receivers, cu_seqlens_q, cu_seqlens_k, qblock_base,
                                   max_seqlen_q, total_q, l_r_range)
    _check(_lib.mf_map_retrieve_multi(arr, len(receivers), _stream(stream)))
    del keep
    return outs


def mf_retrieve_multi_fused(layers, receivers, cu_seqlens_q, cu_seqlens_k, qblock_base,
                            max_seqlen_q, total_q=None, l_r_range=None) -> int:
    arr, keep, _ = _multi_descs(layers, receivers, cu_seqlens_q, cu_seqlens_k, qblock_base,
                                max_seqlen_q, total_q, l_r_range)
    return _lib.mf_retrieve_multi_fused(arr, len(receivers))


def mf_retrieve_path(layers, layer_map, W, V, cu_seqlens_q, cu_seqlens_k, qblock_base,
                     max_seqlen_q, h_r, h_kv, O, paged=None, force_simt=False) -> int:
    h_s, B = layers[0].values.shape[1], layers[0].values.shape[2]
    d, keep = _retrieve_desc(layers, layer_map, (0, len(layer_map)), W, V, O, cu_seqlens_q,
                             cu_seqlens_k, qblock_base, max_seqlen_q, h_s, B, h_r, h_kv, 0, 0,
                             paged, MF_RETRIEVE_FORCE_SIMT if force_simt else 0)
    return _lib.mf_retrieve_path(ctypes.byref(d))


def mf_prefix_hashes(tokens, B: int):
    """uint64 [ceil(L / B)]: FNV-1a 64 of the token bytes of each prefix ending a query block."""
    import numpy as np
    t = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
    n = -(-t.size // B)
    out = np.zeros(n, dtype=np.uint64)
    _check(_lib.mf_prefix_hashes(t.ctypes.data_as(_P), t.size, int(B), out.ctypes.data_as(_P)))
    return out


class BlockCache:
    """Prefix-hash cache of compressed query-block rows in a caller-owned device pool
    (include/mf.h, mf_cache_*)."""

    def __init__(self, pool: torch.Tensor, h_s: int, B: int, dtype=torch.bfloat16):
        self.pool = pool  # keeps the memory alive
        d = CacheDesc(_ptr(pool), pool.numel() * pool.element_size(), int(h_s), int(B),
                      MF_BF16 if dtype == torch.bfloat16 else MF_F32)
        h = _P()
        _check(_lib.mf_cache_create(ctypes.byref(d), ctypes.byref(h)))
        self._h = h

    def close(self):
        if getattr(self, "_h", None):
            _lib.mf_cache_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    def put(self, layer: int, bsr: BSR, hashes, row0: int = 0, nrows: Optional[int] = None,
            row_ptr_host=None, col_idx_host=None, stream=None) -> int:
        """Insert rows [row0, row0 + nrows) of a compressed layer; returns the rows added.
        The BSR's index arrays are read back to the host when not given."""
        import numpy as np
        rp = np.ascontiguousarray(row_ptr_host if row_ptr_host is not None
                                  else bsr.row_ptr.cpu().numpy(), dtype=np.int32)
        ci = np.ascontiguousarray(col_idx_host if col_idx_host is not None
                                  else bsr.col_idx.cpu().numpy(), dtype=np.int32)
        hs = np.ascontiguousarray(hashes, dtype=np.uint64)
        n = len(hs) if nrows is None else nrows
        got = _I64(0)
        d = bsr.desc()
        _check(_lib.mf_cache_put(self._h, int(layer), ctypes.byref(d), rp.ctypes.data_as(_P),
                                 ci.ctypes.data_as(_P), int(row0), int(n), hs.ctypes.data_as(_P),
                                 ctypes.byref(got), _stream(stream)))
        return got.value

    def get(self, layer: int, hashes, out: BSR, stream=None) -> int:
        """Assemble the longest cached prefix of the rows into `out`; returns the rows found."""
        import numpy as np
        hs = np.ascontiguousarray(hashes, dtype=np.uint64)
        hit = _I32(0)
        _check(_lib.mf_cache_get(self._h, int(layer), hs.ctypes.data_as(_P), len(hs),
                                 _ptr(out.row_ptr), _ptr(out.col_idx), _ptr(out.values),
                                 out.capacity, ctypes.byref(hit), _stream(stream)))
        return hit.value

    def stats(self) -> dict:
        import numpy as np
        o = np.zeros(6, dtype=np.int64)
        _check(_lib.mf_cache_stats(self._h, o.ctypes.data_as(_P)))
        return dict(zip(("rows", "used", "free", "hits", "misses", "evicted"), o.tolist()))


def mf_set_wait_limit(limit_ns: int = 0, stall: bool = False) -> None:
    """Limit of every pipeline wait of the tensor-core kernels for later launches (0: the
    default, 2 s); stall=True makes those launches wait on a barrier nothing arrives at, so the
    limit runs out and MF_ERR_TIMEOUT is reported (a test of the timeout path)."""
    _check(_lib.mf_set_wait_limit(int(limit_ns), 1 if stall else 0))


def mf_get_status(stream=None):
    """Synchronise the stream; return (status, bits) of the device status word and clear it."""
    bits = ctypes.c_uint32(0)
    rc = _lib.mf_get_status(_stream(stream), ctypes.byref(bits))
    return rc, bits.value


def check_device_status(stream=None):
    rc, bits = mf_get_status(stream)
    if rc != MF_OK:
        raise MFError(rc, f"{_lib.mf_last_error().decode()} (bits {bits:#x})")


# ----------------------------------------------------------------------------- calibration

def _calib_desc(sender_maps, receiver_maps, seq_offsets, lens, h_s, h_r, B, gram):
    """The host arrays are returned too: they must outlive the call."""
    n = len(lens)
    so = (ctypes.c_int64 * n)(*[int(o[0]) for o in seq_offsets])
    ro = (ctypes.c_int64 * n)(*[int(o[1]) for o in seq_offsets])
    ln = (ctypes.c_int32 * n)(*[int(L) for L in lens])
    d = CalibDesc(_ptr(sender_maps), _ptr(receiver_maps), _dt(sender_maps),
                  ctypes.cast(so, _P), ctypes.cast(ro, _P), ctypes.cast(ln, _P), n, h_s, h_r, B,
                  _ptr(gram))
    return d, (so, ro, ln)


def mf_calib_gram(sender_maps: torch.Tensor, receiver_maps: torch.Tensor, seq_offsets, lens,
                  h_s: int, h_r: int, B: int, gram: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Add the Gram of the stacked sender / receiver maps over the causal positions of every
    sequence to `gram` (float64 [h_s + h_r, h_s + h_r] on the device, created as zeros when
    None).  seq_offsets[s] = (sender element offset, receiver element offset) of sequence s;
    both map tensors are flat, [h][Lp][Lp] per sequence as for mf_compress."""
    if receiver_maps.dtype != sender_maps.dtype:
        raise ValueError("sender and receiver maps must share a dtype")
    F = h_s + h_r
    if gram is None:
        gram = torch.zeros((F, F), dtype=torch.float64, device=sender_maps.device)
    d, keep = _calib_desc(sender_maps, receiver_maps, seq_offsets, lens, h_s, h_r, B, gram)
    nb = ctypes.c_size_t(0)
    _check(_lib.mf_calib_workspace_size(ctypes.byref(d), ctypes.byref(nb)))
    if workspace is None or workspace.numel() < nb.value:
        workspace = torch.empty(max(nb.value, 256), dtype=torch.uint8, device=sender_maps.device)
    _check(_lib.mf_calib_gram(ctypes.byref(d), _ptr(workspace), workspace.numel(), _stream(stream)))
    del keep
    return gram


def mf_calib_path(sender_maps, receiver_maps, seq_offsets, lens, h_s, h_r, B) -> int:
    d, keep = _calib_desc(sender_maps, receiver_maps, seq_offsets, lens, h_s, h_r, B, None)
    d.gram = 16  # any non-null pointer: only the shape is examined
    return _lib.mf_calib_path(ctypes.byref(d))


def mf_calib_solve(gram: torch.Tensor, h_s: int, h_r: int, ridge: float = 0.0, stream=None):
    """Least-squares head map from a Gram: (W float32 [h_r, h_s], residual float64 [h_r]) on the
    device.  A singular sender Gram (ridge 0) is reported by mf_get_status."""
    W = torch.zeros((h_r, h_s), dtype=torch.float32, device=gram.device)
    res = torch.zeros(h_r, dtype=torch.float64, device=gram.device)
    _check(_lib.mf_calib_solve(_ptr(gram), h_s, h_r, float(ridge), _ptr(W), _ptr(res), _stream(stream)))
    return W, res


def choose_sender_layer(residuals_per_candidate: Sequence[torch.Tensor]) -> int:
    """Layer map for one receiver layer: the candidate sender layer whose fitted head map leaves
    the smallest total residual (one residual vector per candidate, from mf_calib_solve)."""
    totals = [float(r.double().sum()) for r in residuals_per_candidate]
    return min(range(len(totals)), key=lambda k: (totals[k], k))
