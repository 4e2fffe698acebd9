"""Pins for oracle.budget: the lemma on a hand-worked example, monotonicity,
and the bound's coverage by simulation."""
import math
import os

import numpy as np
import pytest

from oracle import budget, rng, select, stats


def _rows(golden_dir):
    rows = []
    with open(os.path.join(golden_dir, "clt_budget.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append([float(x) for x in line.split()])
    return rows


def test_lemma_worked_example(golden_dir):
    for n_s, tr, tau, delta, want in _rows(golden_dir):
        assert budget.lemma_budget(n_s, tr, tau, delta) == pytest.approx(want, rel=1e-7)


def test_quantile_textbook_values():
    assert budget.z_two_sided(0.05) == pytest.approx(1.959963984540054, rel=1e-12)
    assert budget.z_two_sided(0.025) == pytest.approx(2.241402727604947, rel=1e-12)


def test_lemma_coverage_by_simulation():
    # draw b per the lemma for a scalar population; the miss rate must stay
    # near or below delta (CLT approximation: allow a small slack)
    r = np.random.default_rng(0)
    pop = r.exponential(size=4000)
    n_s = len(pop)
    s_true = pop.sum()
    tau = 0.02 * s_true
    delta = 0.1
    b = math.ceil(budget.lemma_budget(n_s, pop.var(), tau, delta))
    trials = 3000
    miss = sum(abs(n_s / b * pop[r.integers(0, n_s, b)].sum() - s_true) > tau for _ in range(trials))
    assert miss / trials < delta * 1.3


def _unit(seed, L=2048, d=16, G=4):
    r = np.random.default_rng(seed)
    mu_q = r.standard_normal((G, d))
    k = r.standard_normal(d) + 0.25 * r.standard_normal((L, d))
    v = r.standard_normal((L, d))
    q_ctx = mu_q[:, None] + r.standard_normal((G, L, d))
    q = mu_q + r.standard_normal((G, d))
    return q, k, v, q_ctx


def test_clt_budget_monotone_and_clamped():
    q, k, v, q_ctx = _unit(1)
    L, d = k.shape
    s = 1 / math.sqrt(d)
    st = stats.prefill_stats(q_ctx, k, v, s, "f32")
    blocks, idx, tail = select.select_unit(q, st["blk_mean"], L, 16, 32, 4)
    base = rng.sample_positions(3, 0, 0, 0, tail, 64)
    bs = [budget.clt_budget(q, k, v, idx, base, s, eps, 0.05, len(tail))[0] for eps in (0.4, 0.2, 0.1, 0.05)]
    assert bs == sorted(bs)
    assert all(64 <= b <= len(tail) for b in bs)
    b_loose, _ = budget.clt_budget(q, k, v, idx, base, s, 0.1, 0.2, len(tail))
    b_tight, _ = budget.clt_budget(q, k, v, idx, base, s, 0.1, 0.01, len(tail))
    assert b_loose <= b_tight
