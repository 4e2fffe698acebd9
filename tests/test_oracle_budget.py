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


def _clt_unit(golden_dir):
    """The hand-worked unit of tests/golden/clt_unit.txt as oracle inputs."""
    rows, want, prm = [], {}, {}
    with open(os.path.join(golden_dir, "clt_unit.txt")) as f:
        for line in f:
            t = line.split()
            if not t or t[0].startswith("#"):
                continue
            if t[0] in ("I", "S"):
                rows.append((t[0], int(t[1]), [float(x) for x in t[2:4]], [float(x) for x in t[4:6]]))
            elif t[0] in ("bN", "bD"):
                want[(t[0], int(t[1]) - 1)] = (int(t[2]), int(t[3]))
            elif t[0] == "params":
                prm = {t[i]: float(t[i + 1]) for i in range(1, len(t), 2)}
    n_t = int(prm["n_t"])
    idx = np.array([p for kind, p, _, _ in rows if kind == "I"])
    base = np.array([p for kind, p, _, _ in rows if kind == "S"])
    L = len(idx) + n_t
    k = np.zeros((L, 2))
    v = np.zeros((L, 2))
    for _, p, kr, vr in rows:
        k[p], v[p] = kr, vr
    q = np.eye(2)
    return q, k, v, idx, base, n_t, want, prm


def test_clt_budget_hand_worked_unit(golden_dir):
    # every step of the budget's composition: the n_T / b0 scale-up of the
    # base sample in N_hat and D_hat, unbiased spreads, eps/4 and delta/2 per
    # estimate, both bounds of both heads, the max, the ceiling and the clamp
    q, k, v, idx, base, n_t, want, prm = _clt_unit(golden_dir)
    b, det = budget.clt_budget(q, k, v, idx, base, math.log(2.0), prm["eps"], prm["delta"], n_t)
    z2 = prm["z"] ** 2
    for h in range(2):
        for key, got in (("bN", det["b_N"][h]), ("bD", det["b_D"][h])):
            num, den = want[(key, h)]
            assert got == pytest.approx(z2 * num / den, rel=1e-9), (key, h)
    assert b == int(prm["b"])


def test_clt_budget_clamps_to_the_tail(golden_dir):
    # the same unit with eps 50x tighter: the real budget exceeds n_T and the
    # sample is the whole tail; 1000x looser: the base sample already suffices
    q, k, v, idx, base, n_t, want, prm = _clt_unit(golden_dir)
    s = math.log(2.0)
    assert budget.clt_budget(q, k, v, idx, base, s, prm["eps"] / 50, prm["delta"], n_t)[0] == n_t
    assert budget.clt_budget(q, k, v, idx, base, s, prm["eps"] * 1000, prm["delta"], n_t)[0] == len(base)
