"""Seeded synthetic inputs for tests and benchmarks (CPU recipe + GPU twin).

Only input generation lives here; the method's arithmetic lives in the CUDA
library (`cross_model_attention_mf_b200`) and, independently, in `oracle/`.
"""
import ctypes
import os
import subprocess

import numpy as np
import torch

from . import rng
from .configs import ALL, Workload, chunks, page_table  # noqa: F401
from .maps import gen_maps, gen_normal, gen_v, gen_w, heavy_columns  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmfsynth.so")
_lib = None


def build(force=False):
    src = os.path.join(_HERE, "csrc", "gen_maps.cu")
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(src):
        return _LIB_PATH
    cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-shared", "-Xcompiler", "-fPIC", "-o", _LIB_PATH, src]
    subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.mfsynth_gen_maps.restype = ctypes.c_int
        lib.mfsynth_gen_maps.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_int,
                                         ctypes.c_ulonglong, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_void_p]
        lib.mfsynth_fill_normal.restype = ctypes.c_int
        lib.mfsynth_fill_normal.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong,
                                            ctypes.c_ulonglong, ctypes.c_float, ctypes.c_void_p]
        _lib = lib
    return _lib


def _dt(dtype):
    return (0, torch.float32) if dtype == "f32" else (1, torch.bfloat16)


def gen_maps_gpu(out, L, B, h_s, n_heavy, seed=0, layer=0, seq=0, reading=1, dtype="bf16"):
    """Fill `out` (CUDA tensor viewed as [h_s, Lp, Lp]) with the recipe's maps; only the
    causal blocks are written."""
    code, tdt = _dt(dtype)
    Lp = -(-L // B) * B
    assert out.is_cuda and out.dtype == tdt and out.numel() >= h_s * Lp * Lp
    nh = min(n_heavy, L)
    heavy = np.stack([heavy_columns(seed, layer, seq, s, L, nh) for s in range(h_s)]) \
        if nh > 0 else np.zeros((h_s, 1), dtype=np.int32)
    heavy_t = torch.from_numpy(heavy.astype(np.int32)).to(out.device)
    st = torch.cuda.current_stream(out.device).cuda_stream
    rc = _load().mfsynth_gen_maps(out.data_ptr(), code, L, Lp, B, h_s, heavy_t.data_ptr(),
                                  nh, seed, layer, seq, reading, st)
    if rc != 0:
        raise RuntimeError(f"mfsynth_gen_maps failed: {rc}")
    torch.cuda.current_stream(out.device).synchronize()  # heavy_t lifetime
    return out


def fill_normal_gpu(out, seed, tag, a=0, b=0, scale=1.0):
    code = 0 if out.dtype == torch.float32 else 1
    key = int(rng.stream_key(seed, tag, a, b))
    st = torch.cuda.current_stream(out.device).cuda_stream
    rc = _load().mfsynth_fill_normal(out.data_ptr(), code, out.numel(), key, scale, st)
    if rc != 0:
        raise RuntimeError(f"mfsynth_fill_normal failed: {rc}")
    return out


def gen_v_gpu(T, h_kv, d, seed=0, layer=0, dtype="bf16", device="cuda"):
    _, tdt = _dt(dtype)
    v = torch.empty((T, h_kv, d), dtype=tdt, device=device)
    return fill_normal_gpu(v, seed, rng.TAG_V, layer)
