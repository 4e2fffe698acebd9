"""Adaptive sampling budget (vAttention, Method, key designs 2 and 3).

Lemma (key design 2): to estimate the sum s of n_s vectors r_i from b
uniform draws, s_hat = (n_s / b) sum_{i in sample} r_i, it suffices that
    b >= ( Phi^{-1}(1 - delta/2) * n_s * sqrt(Tr Sigma) / tau )^2
for Pr(||s_hat - s|| > tau) <= delta, Sigma the covariance of the r_i.
tau = eps ||N|| for the numerator and eps D for the denominator; the unknown
Sigma, ||N||, D come from a small base sample.

Lemma 4.2 (key design 3): numerator (eps1, delta1) and denominator
(eps2, delta2), eps2 < 0.5, with b = max(b_D, b_N) give
||N/D - N_hat/D_hat|| <= 2 (eps1 + eps2) ||N/D|| with prob. >= 1-delta1-delta2.

Readings (the page does not print Theorem 4.3's allocation): a user target
(eps, delta) on the output is split evenly, eps1 = eps2 = eps/4 and
delta1 = delta2 = delta/2; the base sample is the first b0 draws of the
unit's stream (reused as the first draws of the final sample); Tr Sigma and
the variance of the denominator terms use the unbiased sample estimates; one
budget per KV head = the max over its query heads; b is clamped to
[b0, n_T].

Parity pins (tests/test_oracle_budget.py): the lemma evaluated on a worked
example by hand (tests/golden/clt_budget.txt); the whole budget of one unit
worked by hand in exact rational arithmetic (tests/golden/clt_unit.txt: the
n_T / b0 scale-up, the unbiased spreads, eps/4 and delta/2, both bounds of
both heads, the max, the ceiling, the clamp); monotonicity in eps / delta;
the bound's coverage checked by simulation.
"""
import math

import numpy as np
from scipy.stats import norm


def z_two_sided(delta):
    """Phi^{-1}(1 - delta/2)."""
    return float(norm.ppf(1.0 - delta / 2.0))


def lemma_budget(n_s, trace_sigma, tau, delta):
    """Smallest real b the lemma asks for (not rounded)."""
    if tau <= 0:
        return math.inf
    return (z_two_sided(delta) * n_s * math.sqrt(max(trace_sigma, 0.0)) / tau) ** 2


def clt_budget(q, k, v, idx, base_pos, scale, eps, delta, n_t):
    """Budget b for one unit (KV head) from a base sample of tail positions.

    q [G, d]; idx = exactly-read positions; base_pos = the b0 base draws.
    Returns (b, details) with b an int in [b0, n_T].
    """
    b0 = len(base_pos)
    if n_t == 0 or b0 < 2:
        return 0, {}
    eps1 = eps2 = eps / 4.0
    d1 = d2 = delta / 2.0
    l_i = scale * (q @ k[idx].T)                         # [G, |I|]
    l_s = scale * (q @ k[base_pos].T)                    # [G, b0]
    m = np.maximum(l_i.max(axis=1) if len(idx) else -np.inf, l_s.max(axis=1))
    e_i = np.exp(l_i - m[:, None])
    e_s = np.exp(l_s - m[:, None])
    n_hat = e_i @ v[idx] + (n_t / b0) * (e_s @ v[base_pos])   # [G, d]
    d_hat = e_i.sum(axis=1) + (n_t / b0) * e_s.sum(axis=1)    # [G]
    best = 0.0
    det = {"b_N": [], "b_D": []}
    for h in range(q.shape[0]):
        r = e_s[h][:, None] * v[base_pos]                   # numerator terms [b0, d]
        tr = float(r.var(axis=0, ddof=1).sum())
        var_d = float(e_s[h].var(ddof=1))
        b_n = lemma_budget(n_t, tr, eps1 * float(np.linalg.norm(n_hat[h])), d1)
        b_d = lemma_budget(n_t, var_d, eps2 * float(d_hat[h]), d2)
        det["b_N"].append(b_n)
        det["b_D"].append(b_d)
        best = max(best, b_n, b_d)
    b = int(min(max(math.ceil(best) if math.isfinite(best) else n_t, b0), n_t))
    return b, det
