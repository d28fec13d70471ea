"""Device-side layout of a synthetic workload: packed maps, V (contiguous or paged), W and
the varlen / chunk metadata tensors.  Input plumbing only (no method arithmetic)."""
from dataclasses import dataclass
from typing import List, Optional, Tuple

import numpy as np
import torch

from . import gen_maps_gpu, gen_normal, page_table, rng
from .configs import Workload
from .maps import gen_maps, gen_w


def _tdt(dtype):
    return torch.float32 if dtype == "f32" else torch.bfloat16


@dataclass
class MapPack:
    maps: torch.Tensor            # flat, device
    map_seq_offset: torch.Tensor  # int64 [nseq], device
    cu_seqlens: torch.Tensor      # int32 [nseq + 1], device
    offsets: List[int]            # host copy of map_seq_offset
    lens: List[int]

    def seq_view(self, s: int, h_s: int, B: int) -> torch.Tensor:
        L = self.lens[s]
        Lp = -(-L // B) * B
        o = self.offsets[s]
        return self.maps[o:o + h_s * Lp * Lp].view(h_s, Lp, Lp)


def map_offsets(w: Workload) -> Tuple[List[int], int]:
    offs, o = [], 0
    for Lp in w.Lp:
        offs.append(o)
        o += w.h_s * Lp * Lp
    return offs, o


def alloc_maps(w: Workload, device="cuda") -> MapPack:
    offs, total = map_offsets(w)
    maps = torch.empty(total, dtype=_tdt(w.dtype), device=device)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(w.lens)]), dtype=torch.int32, device=device)
    return MapPack(maps, torch.tensor(offs, dtype=torch.int64, device=device), cu, offs, list(w.lens))


def fill_maps(pack: MapPack, w: Workload, layer: int, use_gpu: bool = True) -> MapPack:
    """The recipe's maps of sender layer `layer` for every sequence of the pack."""
    for s, L in enumerate(w.lens):
        view = pack.seq_view(s, w.h_s, w.B)
        if use_gpu:
            gen_maps_gpu(view, L, w.B, w.h_s, w.n_heavy, seed=w.seed, layer=layer, seq=s,
                         reading=w.reading, dtype=w.dtype)
        else:
            view.copy_(gen_maps(L, w.B, w.h_s, w.n_heavy, seed=w.seed, layer=layer, seq=s,
                                reading=w.reading, dtype=w.dtype).to(view.device))
    return pack


def w_weights(w: Workload, device="cuda") -> torch.Tensor:
    return gen_w(w.n_receiver_layers, w.h_r, w.h_s, seed=w.seed).to(device)


def v_contiguous(w: Workload, layer: int, device="cuda", use_gpu: bool = True) -> torch.Tensor:
    """Receiver V [T, h_kv, d] of receiver layer `layer` (counter over the packed tokens)."""
    T = w.tokens
    if use_gpu:
        from . import fill_normal_gpu
        v = torch.empty((T, w.h_kv, w.d), dtype=_tdt(w.dtype), device=device)
        return fill_normal_gpu(v, w.seed, rng.TAG_V, layer)
    z = gen_normal(T * w.h_kv * w.d, w.seed, rng.TAG_V, layer).reshape(T, w.h_kv, w.d)
    return torch.from_numpy(z).to(_tdt(w.dtype)).to(device)


def v_paged(w: Workload, v: torch.Tensor):
    """Scatter a contiguous V into the workload's shuffled pages.
    Returns (V_paged [n_pages, page, h_kv, d], block_table int32 [nseq, max_pages])."""
    table, npages = page_table(w)
    ps = w.page_size
    vp = torch.zeros((npages, ps, w.h_kv, w.d), dtype=v.dtype, device=v.device)
    tab = torch.from_numpy(table).to(v.device)
    start = 0
    for s, L in enumerate(w.lens):
        n = -(-L // ps)
        pad = n * ps - L
        src = v[start:start + L]
        if pad:
            src = torch.cat([src, torch.zeros((pad, w.h_kv, w.d), dtype=v.dtype, device=v.device)])
        vp[tab[s, :n].long()] = src.view(n, ps, w.h_kv, w.d)
        start += L
    return vp, tab


def qblock_base(w: Workload, device="cuda") -> torch.Tensor:
    return torch.tensor(np.concatenate([[0], np.cumsum(w.nqb)[:-1]]), dtype=torch.int32, device=device)


def step_tensors(step, device="cuda"):
    """cu_seqlens_q / cu_seqlens_k (int32, device) and max q_len of one chunked-prefill step
    [(q_len, k_len)].  A contiguous V must hold each sequence's k_len-token prefix packed in
    the same order (key j of sequence s at token cu_seqlens_k[s] + j)."""
    q, k = [0], [0]
    for ql, kl in step:
        q.append(q[-1] + ql)
        k.append(k[-1] + kl)
    return (torch.tensor(q, dtype=torch.int32, device=device),
            torch.tensor(k, dtype=torch.int32, device=device), max(ql for ql, _ in step))


def pack_prefixes(v: torch.Tensor, lens, step) -> torch.Tensor:
    """Contiguous V of one step: the k_len-token prefix of every sequence, packed."""
    starts = np.concatenate([[0], np.cumsum(lens)])
    return torch.cat([v[starts[s]:starts[s] + kl] for s, (_, kl) in enumerate(step)])
