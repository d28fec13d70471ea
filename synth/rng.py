"""Counter-based random numbers shared by every seeded input of this repository.

This module holds no part of the method's arithmetic: it only turns
(seed, tensor tag, indices, counter) into bits, uniforms and normals.

Generator: SplitMix64 (G. L. Steele, D. Lea, C. H. Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014).  The n-th output of the
stream that starts at state `key` is mix64(key + (n + 1) * GAMMA), which makes
every draw addressable by its counter.  The CUDA map generator in
`synth/csrc/gen_maps.cu` implements the same definition on its own.

Normals: Box-Muller (G. E. P. Box, M. E. Muller, Ann. Math. Stat. 1958) in
float32 from two 24-bit uniforms: u1 in (0, 1], u2 in [0, 1).
"""
import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# tensor tags (part of the stream key)
TAG_NOISE = 1      # map logit noise, one stream per (layer, seq, sender head)
TAG_HEAVY = 2      # heavy-column draws, one stream per (layer, seq, sender head)
TAG_V = 3          # receiver V, one stream per receiver layer
TAG_W = 4          # head-mapping weights, one stream for all receiver layers
TAG_LENS = 5       # varlen sequence lengths
TAG_PAGES = 6      # page permutation of a paged V cache


def mix64(z):
    """SplitMix64 output function on uint64 (scalar or array), wrapping mod 2**64."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed, tag, a=0, b=0, c=0):
    """Key of one stream: fold (tag, a, b, c) into the seed, one mix64 per field."""
    k = np.uint64(seed)
    with np.errstate(over="ignore"):
        for f in (tag, a, b, c):
            k = mix64(k ^ (np.uint64(f + 1) * GAMMA))
    return np.uint64(k)


def draw(key, n):
    """n-th SplitMix64 output (n: int or uint64 array) of the stream at `key`."""
    n = np.asarray(n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(np.uint64(key) + (n + np.uint64(1)) * GAMMA)


def below(x, m):
    """Map 64-bit draws to integers in [0, m) by multiply-shift on the top 32 bits."""
    x = np.asarray(x, dtype=np.uint64)
    return ((x >> np.uint64(32)) * np.uint64(m)) >> np.uint64(32)


def normal(key, n):
    """Standard normals (float32) for counters n: Box-Muller on draws 2n and 2n+1."""
    n = np.asarray(n, dtype=np.uint64)
    x0 = draw(key, np.uint64(2) * n)
    x1 = draw(key, np.uint64(2) * n + np.uint64(1))
    scale = np.float32(2.0 ** -24)
    u1 = ((x0 >> np.uint64(40)).astype(np.float32) + np.float32(1.0)) * scale
    u2 = (x1 >> np.uint64(40)).astype(np.float32) * scale
    r = np.sqrt(np.float32(-2.0) * np.log(u1))
    return (r * np.cos(np.float32(2.0 * np.pi) * u2)).astype(np.float32)
