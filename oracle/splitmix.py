"""Counter-based permutation draws for merge-then-reinitialize.

TEST INFRASTRUCTURE ONLY (see the package header).

The pages resample the permutations at each merge ("Reparameterized LLM
Training via Orthogonal Equivalence Transformation", §3 Merge-then-Reinitialize)
but fix no generator.  The library and this oracle each implement the same
published generator, SplitMix64 (Steele, Lea and Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014; the 64-bit finaliser with
constants 0xbf58476d1ce4e5b9 / 0x94d049bb133111eb and increment
0x9e3779b97f4a7c15), used counter-style:

  out(s, i)      = mix(s + (i + 1) * 0x9e3779b97f4a7c15)   (the i-th output of
                   the stream whose state starts at s)
  stream(seed,l) = out(seed, l)        (l = 0 for R, 1 for P)
  key_l[i]       = out(stream(seed, l), i)
  pi_l           = the indices sorted by (key_l[i], i) ascending

so pi_l[r] is the index whose key has rank r.  All arithmetic is modulo 2^64.
"""
from __future__ import annotations

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
C1 = 0xBF58476D1CE4E5B9
C2 = 0x94D049BB133111EB
MASK = (1 << 64) - 1


def mix64(z: int) -> int:
    z &= MASK
    z = ((z ^ (z >> 30)) * C1) & MASK
    z = ((z ^ (z >> 27)) * C2) & MASK
    return z ^ (z >> 31)


def splitmix_output(state: int, i: int) -> int:
    """The i-th (0-based) output of SplitMix64 started from `state`."""
    return mix64((state + (i + 1) * GAMMA) & MASK)


def splitmix_stream(state: int, count: int):
    """Sequential form of the generator (state += gamma; return mix(state))."""
    s = state & MASK
    out = []
    for _ in range(count):
        s = (s + GAMMA) & MASK
        out.append(mix64(s))
    return out


def permutation_keys(seed: int, lane: int, n: int) -> np.ndarray:
    s = splitmix_output(seed & MASK, lane)
    return np.array([splitmix_output(s, i) for i in range(n)], dtype=np.uint64)


def resample_permutation(seed: int, lane: int, n: int) -> np.ndarray:
    keys = permutation_keys(seed, lane, n)
    # stable sort on the key == sort by (key, index)
    return np.argsort(keys, kind="stable").astype(np.int32)
