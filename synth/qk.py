"""Seeded synthetic sender queries and keys (CPU torch), the input of compression from Q, K.

Recipe, for one layer of a varlen pack (T tokens; per sequence, positions restart at 0):

    Q[t, s, :] = rope(pos) (dims 0..2P-1)  +  noise * z_q  +  c * u_g        (dims 2P..d-1)
    K[t, g, :] = rope(pos)                 +  noise * z_k
                 + (SINK * sqrt(d) / c) * u_g   if pos < 4            (attention sinks)
                 + (HEAVY * sqrt(d) / c) * u_g  if pos is a heavy key of (sequence, g)

with g = s * h_kv // h_s, rope(pos) = a (cos(w_k pos), sin(w_k pos)), k < P = 16,
w_k = 10000^(-k / P), a = sqrt(RECENCY * sqrt(d) / P), u_g a random unit vector (one per key
head) in the non-positional dims, z ~ N(0, 1).  With the scale 1 / sqrt(d) the scaled score of
query i and key j is about RECENCY * mean_k cos(w_k (i - j)) + SINK / HEAVY bonuses + noise.
The recency peak dominates (the last 8 keys hold 60-99% of a row's mass at 300-1000 tokens);
sinks and heavy keys take a few percent.  At L = 8192 and tau = 0.95, about 3% of the causal
blocks are kept (11% at 4096).  Rounded to the requested dtype.  Nothing here computes a
softmax, a mass or a selection.
"""
import numpy as np
import torch

P = 16
BASE = 10000.0
RECENCY = 20.0
SINK = 10.0
HEAVY = 8.0
NOISE = 0.7
C = 4.0
SINK_TOKENS = 4


def gen_qk(lens, h_s, h_kv, d, n_heavy=16, seed=0, layer=0, dtype=torch.bfloat16):
    """(Q [T, h_s, d], K [T, h_kv, d]) on the CPU for sequences of lengths `lens`."""
    assert h_s % h_kv == 0 and d > 2 * P
    g = torch.Generator().manual_seed(int(seed) * 1000003 + int(layer) * 7919 + 17)
    T = int(sum(lens))
    dn = d - 2 * P
    sd = float(np.sqrt(d))
    a = float(np.sqrt(RECENCY * sd / P))
    u = torch.randn(h_kv, dn, generator=g, dtype=torch.float64)
    u = u / u.norm(dim=1, keepdim=True)
    pos = torch.cat([torch.arange(L, dtype=torch.float64) for L in lens])
    w = BASE ** (-torch.arange(P, dtype=torch.float64) / P)
    ang = pos[:, None] * w[None, :]
    rope = a * torch.cat([torch.cos(ang), torch.sin(ang)], dim=1)      # [T, 2P]
    Q = torch.empty(T, h_s, d, dtype=torch.float64)
    K = torch.empty(T, h_kv, d, dtype=torch.float64)
    Q[:, :, :2 * P] = rope[:, None, :]
    K[:, :, :2 * P] = rope[:, None, :]
    Q[:, :, 2 * P:] = NOISE * torch.randn(T, h_s, dn, generator=g, dtype=torch.float64)
    K[:, :, 2 * P:] = NOISE * torch.randn(T, h_kv, dn, generator=g, dtype=torch.float64)
    grp = torch.arange(h_s) * h_kv // h_s
    Q[:, :, 2 * P:] += C * u[grp][None, :, :]
    start = 0
    for L in lens:
        K[start:start + min(L, SINK_TOKENS), :, 2 * P:] += (SINK * sd / C) * u[None, :, :]
        for kv in range(h_kv):
            nh = min(n_heavy, L)
            heavy = torch.randperm(L, generator=g)[:nh] + start
            K[heavy, kv, 2 * P:] += (HEAVY * sd / C) * u[kv][None, :]
        start += L
    return Q.to(dtype), K.to(dtype)
