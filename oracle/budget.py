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

Two further budget rules the page names without printing them:
  * Theorem 4.3 allocates the output target over (eps1, eps2, delta1,
    delta2) by a minimisation; reading: 2 (eps1 + eps2) = eps, delta1 +
    delta2 = delta, eps1 = f eps/2, delta1 = g delta with f and g on the grid
    1/20, 2/20, ..., 19/20 (eps2 < 0.5 required), and b = the smallest over
    the grid of max over heads of max(b_N(eps1, delta1), b_D(eps2, delta2));
    ties go to the first grid point in (f, g) order.  The even split (f = g =
    1/2) is a grid point, so the search never asks for more.
  * the conservative Hoeffding version (the page's appendix remark): for
    iid terms in a range of width R, Pr(|mean - mu| >= t) <= 2 exp(-2 b t^2 /
    R^2), so b >= R^2 n_s^2 ln(2/delta) / (2 tau^2); the ranges are not known
    in advance, so (as the CLT version does with the variance) they are the
    base sample's max - min; the numerator is a vector, bounded coordinate
    by coordinate (each within tau / sqrt(d) with probability delta1 / d, a
    union bound): b_N = d n_s^2 ln(2 d / delta1) max_e R_e^2 / (2 tau_N^2).
    eps and delta split evenly as in clt_budget.

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


def _estimates(q, k, v, idx, base_pos, scale, n_t):
    """N_hat [G, d], D_hat [G] and the base sample's terms: e [G, b0] and
    e V [G, b0, d], all relative to one common shift (it cancels from every
    budget)."""
    b0 = len(base_pos)
    l_i = scale * (q @ k[idx].T)
    l_s = scale * (q @ k[base_pos].T)
    m = np.maximum(l_i.max(axis=1) if len(idx) else -np.inf, l_s.max(axis=1))
    e_i = np.exp(l_i - m[:, None])
    e_s = np.exp(l_s - m[:, None])
    n_hat = e_i @ v[idx] + (n_t / b0) * (e_s @ v[base_pos])
    d_hat = e_i.sum(axis=1) + (n_t / b0) * e_s.sum(axis=1)
    r = e_s[:, :, None] * v[base_pos][None, :, :]
    return n_hat, d_hat, e_s, r


def _clamp(best, b0, n_t):
    return int(min(max(math.ceil(best) if math.isfinite(best) else n_t, b0), n_t))


GRID = tuple(i / 20.0 for i in range(1, 20))


def clt_budget_search(q, k, v, idx, base_pos, scale, eps, delta, n_t):
    """The CLT budget with the (eps, delta) allocation searched over the grid
    (reading of Theorem 4.3, module docstring).  Returns (b, details) with
    the chosen split f, g and the real-valued budget there."""
    b0 = len(base_pos)
    if n_t == 0 or b0 < 2:
        return 0, {}
    n_hat, d_hat, e_s, r = _estimates(q, k, v, idx, base_pos, scale, n_t)
    G = q.shape[0]
    tr = [float(r[h].var(axis=0, ddof=1).sum()) for h in range(G)]
    vd = [float(e_s[h].var(ddof=1)) for h in range(G)]
    best = (math.inf, None, None)
    for f in GRID:
        eps1, eps2 = f * eps / 2.0, (1.0 - f) * eps / 2.0
        if eps2 >= 0.5:
            continue
        for g in GRID:
            d1, d2 = g * delta, (1.0 - g) * delta
            b = 0.0
            for h in range(G):
                b = max(b, lemma_budget(n_t, tr[h], eps1 * float(np.linalg.norm(n_hat[h])), d1),
                        lemma_budget(n_t, vd[h], eps2 * float(d_hat[h]), d2))
            if b < best[0]:
                best = (b, f, g)
    return _clamp(best[0], b0, n_t), {"b_real": best[0], "f": best[1], "g": best[2]}


def hoeffding_budget(q, k, v, idx, base_pos, scale, eps, delta, n_t):
    """The conservative Hoeffding budget (module docstring), eps and delta
    split evenly between numerator and denominator."""
    b0 = len(base_pos)
    if n_t == 0 or b0 < 2:
        return 0, {}
    n_hat, d_hat, e_s, r = _estimates(q, k, v, idx, base_pos, scale, n_t)
    G, d = q.shape[0], v.shape[1]
    eps1 = eps2 = eps / 4.0
    d1 = d2 = delta / 2.0
    det = {"b_N": [], "b_D": []}
    best = 0.0
    for h in range(G):
        rn2 = float(((r[h].max(axis=0) - r[h].min(axis=0)) ** 2).max())
        rd2 = float((e_s[h].max() - e_s[h].min()) ** 2)
        tn = eps1 * float(np.linalg.norm(n_hat[h]))
        td = eps2 * float(d_hat[h])
        b_n = d * n_t ** 2 * math.log(2.0 * d / d1) * rn2 / (2.0 * tn ** 2) if tn > 0 else math.inf
        b_d = n_t ** 2 * math.log(2.0 / d2) * rd2 / (2.0 * td ** 2) if td > 0 else math.inf
        det["b_N"].append(b_n)
        det["b_D"].append(b_d)
        best = max(best, b_n, b_d)
    return _clamp(best, b0, n_t), det


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
