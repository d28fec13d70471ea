"""The five synthetic workloads (shapes, dtypes, value recipe, seed).

They stand in for the pages' model pairs (Qwen3, Ministral3) and for the
LMSYS / ShareGPT4 routing traces, which are not available here: every tensor
is drawn from the seeded recipe in `synth.maps`.

Notation follows the MapFlow pages: h_s sender heads, h_r receiver heads,
h_kv receiver KV heads (GQA), d head dim, B block size, tau the cumulative
attention-probability threshold.
"""
from dataclasses import dataclass, field, replace
from typing import List, Optional, Tuple

import numpy as np

from . import rng


@dataclass(frozen=True)
class Workload:
    name: str
    lens: Tuple[int, ...]          # sequence lengths of the varlen pack
    B: int                          # block size
    h_s: int                        # sender heads
    h_r: int                        # receiver heads
    h_kv: int                       # receiver KV heads
    d: int                          # head dim
    dtype: str                      # "f32" or "bf16" (maps, V, O)
    tau: float
    n_heavy: int                    # heavy columns per (layer, seq, sender head)
    n_sender_layers: int = 1
    n_receiver_layers: int = 1
    chunk: int = 0                  # query chunk of chunked prefill (0 = whole sequence)
    page_size: int = 0              # paged V page (0 = contiguous V)
    reading: int = 1                # map-generator reading: 1 (literal sum) or 3 (bonuses exempt from decay)
    seed: int = 0

    @property
    def Lp(self) -> List[int]:
        return [-(-L // self.B) * self.B for L in self.lens]

    @property
    def nqb(self) -> List[int]:
        return [-(-L // self.B) for L in self.lens]

    @property
    def causal_blocks(self) -> int:
        return sum(n * (n + 1) // 2 for n in self.nqb)

    @property
    def tokens(self) -> int:
        return sum(self.lens)

    def layer_map(self) -> List[int]:
        """Receiver layer -> sender layer: l_s = round(l_r * (S-1)/(R-1)), no .5 ties for the
        Qwen-like pair (40 -> 36 gives floor((78*l_r + 35) / 70))."""
        S, R = self.n_sender_layers, self.n_receiver_layers
        if R == 1:
            return [0]
        # exact rational rounding: floor((2*(S-1)*l + (R-1)) / (2*(R-1)))
        return [(2 * (S - 1) * l + (R - 1)) // (2 * (R - 1)) for l in range(R)]

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


def _c5_lens(seed: int, n: int = 16, lo: int = 1024, hi: int = 8192) -> Tuple[int, ...]:
    key = rng.stream_key(seed, rng.TAG_LENS)
    x = rng.draw(key, np.arange(n, dtype=np.uint64))
    return tuple(int(lo + v) for v in rng.below(x, hi - lo + 1))


TINY = Workload("tiny", (256,), B=32, h_s=4, h_r=2, h_kv=1, d=64, dtype="f32",
                tau=0.9, n_heavy=3)
MINISTRAL_PAIR = Workload("ministral_pair", (8192,), B=64, h_s=32, h_r=32, h_kv=8, d=128,
                          dtype="bf16", tau=0.95, n_heavy=16)
QWEN_PAIR = Workload("qwen_pair", (2048, 4096, 6144, 4096), B=64, h_s=40, h_r=32, h_kv=8,
                     d=128, dtype="bf16", tau=0.95, n_heavy=16,
                     n_sender_layers=40, n_receiver_layers=36)
LONG_CONTEXT = Workload("long_context", (32768,), B=128, h_s=32, h_r=24, h_kv=8, d=128,
                        dtype="bf16", tau=0.95, n_heavy=8)
ROUTING_BATCH = Workload("routing_batch", _c5_lens(0), B=64, h_s=32, h_r=32, h_kv=8, d=128,
                         dtype="bf16", tau=0.95, n_heavy=16, chunk=2048, page_size=16)

ALL = {w.name: w for w in (TINY, MINISTRAL_PAIR, QWEN_PAIR, LONG_CONTEXT, ROUTING_BATCH)}

LONG_CONTEXT_SWEEP = [(tau, heavy) for heavy in (8, 64) for tau in (0.8, 0.9, 0.95, 0.99)]


def chunks(w: Workload) -> List[List[Tuple[int, int]]]:
    """Chunked-prefill schedule: step k holds, per sequence still running, (q_len, k_len):
    the queries are the last q_len tokens of the k_len-token prefix."""
    if w.chunk <= 0:
        return [[(L, L) for L in w.lens]]
    steps = []
    k = 0
    while True:
        step = []
        for L in w.lens:
            start = k * w.chunk
            if start < L:
                end = min(start + w.chunk, L)
                step.append((end - start, end))
            else:
                step.append((0, 0))
        if all(q == 0 for q, _ in step):
            return steps
        steps.append(step)
        k += 1


def page_table(w: Workload, lens=None) -> Tuple[np.ndarray, int]:
    """Shuffled block table of a paged V cache: int32 [nseq, max_pages], unused slots -1,
    and the total page count.  The permutation is a Fisher-Yates shuffle driven by the
    TAG_PAGES stream."""
    lens = list(w.lens if lens is None else lens)
    ps = w.page_size
    npages = [-(-L // ps) for L in lens]
    total = sum(npages)
    key = rng.stream_key(w.seed, rng.TAG_PAGES)
    perm = np.arange(total, dtype=np.int64)
    x = rng.draw(key, np.arange(max(total - 1, 0), dtype=np.uint64))
    for t, i in enumerate(range(total - 1, 0, -1)):
        j = int(rng.below(x[t], i + 1))
        perm[i], perm[j] = perm[j], perm[i]
    table = np.full((len(lens), max(npages)), -1, dtype=np.int32)
    base = 0
    for s, n in enumerate(npages):
        table[s, :n] = perm[base:base + n]
        base += n
    return table, total
