"""Seeded synthetic sender attention maps, receiver V and head-mapping W (CPU, numpy).

Map recipe (one (layer, sequence, sender head) at a time), for query row i and key j <= i:

    logit[i, j] = (bonus[j] + decay[i, j]) + z[i, j]                         (float32)
    bonus[j]    = 2.0 * [j < 4]  +  1.5 * [j is a heavy column]
    decay[i, j] = -0.05 * (i - j)                 reading 1: applied to every key
                  -0.05 * (i - j) * [j not sink and not heavy]   reading 3
    z[i, j]     ~ N(0, 1), counter i * Lp + j of the TAG_NOISE stream

and the map row is the causal softmax of that row (subtract the row max, exp, divide
by the sum), rounded to the map dtype.  Entries with j > i, and every entry of a
padding row i >= L, are 0.  Heavy columns are min(n_heavy, L) distinct keys drawn
uniformly from [0, L) (rejection of repeats, TAG_HEAVY stream).

Nothing here computes block statistics, selection, head mixing or P.V: this module
only makes inputs.  `synth/csrc/gen_maps.cu` follows the same recipe on the GPU for
the sizes that do not fit a CPU run; the two agree up to float32 rounding of
exp/log/cos.
"""
import numpy as np
import torch

from . import rng

SINK_TOKENS = 4
SINK_BONUS = 2.0
HEAVY_BONUS = 1.5
DECAY = 0.05


def heavy_columns(seed, layer, seq, head, L, n_heavy):
    """min(n_heavy, L) distinct heavy columns of one (layer, sequence, sender head)."""
    n_heavy = min(n_heavy, L)
    key = rng.stream_key(seed, rng.TAG_HEAVY, layer, seq, head)
    chosen, seen, n = [], set(), 0
    while len(chosen) < n_heavy:
        # draw in batches; the accepted sequence is the same as one-at-a-time
        xs = rng.below(rng.draw(key, np.arange(n, n + 64, dtype=np.uint64)), L)
        n += 64
        for c in xs.tolist():
            if c not in seen:
                seen.add(c)
                chosen.append(c)
                if len(chosen) == n_heavy:
                    break
    return np.array(chosen, dtype=np.int32)


def logits_rows(seed, layer, seq, head, L, Lp, rows, heavy, reading=1):
    """float32 logits [len(rows), Lp] of the given query rows (valid where j <= i < L)."""
    key = rng.stream_key(seed, rng.TAG_NOISE, layer, seq, head)
    i = np.asarray(rows, dtype=np.int64)[:, None]
    j = np.arange(Lp, dtype=np.int64)[None, :]
    z = rng.normal(key, (i * Lp + j).astype(np.uint64))
    sink = j < SINK_TOKENS
    hv = np.zeros(Lp, dtype=bool)
    hv[np.asarray(heavy, dtype=np.int64)] = True
    hv = hv[None, :]
    bonus = (np.float32(SINK_BONUS) * sink.astype(np.float32)
             + np.float32(HEAVY_BONUS) * hv.astype(np.float32))
    decay = np.float32(-DECAY) * (i - j).astype(np.float32)
    if reading == 3:
        decay = np.where(sink | hv, np.float32(0.0), decay)
    elif reading != 1:
        raise ValueError("reading must be 1 or 3")
    return ((bonus + decay) + z).astype(np.float32)


def causal_softmax_rows(logits, rows, L):
    rows = np.asarray(rows, dtype=np.int64)
    Lp = logits.shape[1]
    j = np.arange(Lp)[None, :]
    valid = (j <= rows[:, None]) & (rows[:, None] < L)
    x = np.where(valid, logits, np.float32(-np.inf))
    m = np.max(np.where(valid, logits, np.float32(-np.inf)), axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, np.float32(0.0))
    e = np.where(valid, np.exp(x - m), np.float32(0.0)).astype(np.float32)
    s = e.sum(axis=1, keepdims=True, dtype=np.float32)
    s = np.where(s > 0, s, np.float32(1.0))
    return (e / s).astype(np.float32)


def gen_maps(L, B, h_s, n_heavy, seed=0, layer=0, seq=0, reading=1, dtype="f32"):
    """Dense maps [h_s, Lp, Lp] (torch, CPU) of one sequence of one sender layer."""
    Lp = -(-L // B) * B
    out = np.zeros((h_s, Lp, Lp), dtype=np.float32)
    rows = np.arange(Lp)
    for s in range(h_s):
        hv = heavy_columns(seed, layer, seq, s, L, n_heavy)
        lg = logits_rows(seed, layer, seq, s, L, Lp, rows, hv, reading)
        out[s] = causal_softmax_rows(lg, rows, L)
    t = torch.from_numpy(out)
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def gen_normal(n, seed, tag, a=0, b=0, scale=1.0):
    key = rng.stream_key(seed, tag, a, b)
    z = rng.normal(key, np.arange(n, dtype=np.uint64))
    if scale != 1.0:
        z = (z * np.float32(scale)).astype(np.float32)
    return z


def gen_v(T, h_kv, d, seed=0, layer=0, dtype="f32"):
    """Receiver V [T, h_kv, d] ~ N(0, 1): counter (t * h_kv + g) * d + c of TAG_V, layer."""
    t = torch.from_numpy(gen_normal(T * h_kv * d, seed, rng.TAG_V, layer).reshape(T, h_kv, d))
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def gen_w(L_r, h_r, h_s, seed=0):
    """Head-mapping weights W [L_r, h_r, h_s] float32 ~ N(0, 1/h_s) (variance 1/h_s)."""
    z = gen_normal(L_r * h_r * h_s, seed, rng.TAG_W, scale=float(1.0 / np.sqrt(h_s)))
    return torch.from_numpy(z.reshape(L_r, h_r, h_s))
