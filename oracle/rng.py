"""Counter-based draws for the sampling estimator (SplitMix64).

The sampling estimator of vAttention (Method, key design 1) draws tail
indices uniformly at random.  To let the GPU and this oracle draw the SAME
indices without shipping random numbers around, both implement SplitMix64
(G. Steele, D. Lea, C. Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014; the 64-bit finaliser constants of S. Vigna's
public-domain splitmix64.c) from its published definition, independently:

  next(state):  state += 0x9E3779B97F4A7C15
                z = state
                z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
                z = (z ^ (z >> 27)) * 0x94D049BB133111EB
                return z ^ (z >> 31)

Stream of unit (sequence b, KV head g) at decode step t (all mod 2**64):
  key = out(out(out(out(seed) ^ b) ^ g) ^ t), with out(x) = mix(x + GAMMA),
  the first output of a SplitMix64 generator whose state is x;
  draw i = out(key + i*GAMMA), the (i+1)-th output of a generator seeded key;
  rank  = ((draw >> 32) * n_T) >> 32   (multiply-shift onto [0, n_T),
          D. Lemire 2019; bias below n_T / 2**32).
Draws are with replacement; rank r maps to the r-th tail position in
ascending order.

Pinned in tests/test_oracle_rng.py against SplitMix64's published first
outputs for seed 0, and by a chi-square test of the ranks.
"""
import numpy as np

MASK = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15


def mix64(z):
    z &= MASK
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK
    return z ^ (z >> 31)


def out(x):
    """First output of a SplitMix64 generator whose state is x."""
    return mix64((x + GAMMA) & MASK)


def unit_key(seed, b, g, step):
    k = out(seed & MASK)
    k = out(k ^ (b & MASK))
    k = out(k ^ (g & MASK))
    k = out(k ^ (step & MASK))
    return k


def draw(key, i):
    return out((key + i * GAMMA) & MASK)


def rank(x, n):
    return ((x >> 32) * n) >> 32


def sample_positions(seed, b, g, step, tail, n_draws):
    """n_draws tail positions, with replacement, in draw order."""
    n = len(tail)
    if n == 0 or n_draws <= 0:
        return np.zeros(0, dtype=np.int64)
    key = unit_key(seed, b, g, step)
    r = [rank(draw(key, i), n) for i in range(n_draws)]
    return np.asarray(tail, dtype=np.int64)[np.asarray(r, dtype=np.int64)]
