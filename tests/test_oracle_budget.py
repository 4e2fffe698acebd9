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
            elif t[0] in ("bN", "bD", "hN", "hD"):
                want[(t[0], int(t[1]) - 1)] = (int(t[2]), int(t[3]))
            elif t[0] == "params":
                prm = {t[i]: float(t[i + 1]) for i in range(1, len(t), 2)}
            elif t[0] == "hoeffding":
                prm.update({"h_" + t[i]: float(t[i + 1]) for i in range(1, len(t), 2)})
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


def test_hoeffding_hand_worked_unit(golden_dir):
    # the Hoeffding budget of the same unit: base-sample ranges of e and of
    # each coordinate of e V, the union bound over the d coordinates, the
    # even eps / delta split, the max over heads and bounds, the ceiling
    q, k, v, idx, base, n_t, want, prm = _clt_unit(golden_dir)
    b, det = budget.hoeffding_budget(q, k, v, idx, base, math.log(2.0), prm["h_eps"], prm["h_delta"], n_t)
    for h in range(2):
        num, den = want[("hN", h)]
        assert det["b_N"][h] == pytest.approx(math.log(80.0) * num / den, rel=1e-9)
        num, den = want[("hD", h)]
        assert det["b_D"][h] == pytest.approx(math.log(40.0) * num / den, rel=1e-9)
    assert b == int(prm["h_b"])


def test_clt_search_never_above_the_even_split(golden_dir):
    # the even split is a grid point, so the searched budget is at most the
    # even-split one; on the hand-worked unit strictly less (1138 there)
    q, k, v, idx, base, n_t, want, prm = _clt_unit(golden_dir)
    s = math.log(2.0)
    b_s, det = budget.clt_budget_search(q, k, v, idx, base, s, prm["eps"], prm["delta"], n_t)
    assert b_s < int(prm["b"]) and det["f"] != 0.5
    for seed in range(4):
        qq, kk, vv, q_ctx = _unit(10 + seed)
        L, d = kk.shape
        st = stats.prefill_stats(q_ctx, kk, vv, 1 / math.sqrt(d), "f32")
        blocks, idx2, tail = select.select_unit(qq, st["blk_mean"], L, 16, 32, 4)
        b0 = rng.sample_positions(seed, 0, 0, 0, tail, 64)
        for eps in (0.1, 0.3):
            even = budget.clt_budget(qq, kk, vv, idx2, b0, 1 / math.sqrt(d), eps, 0.05, len(tail))[0]
            srch = budget.clt_budget_search(qq, kk, vv, idx2, b0, 1 / math.sqrt(d), eps, 0.05, len(tail))[0]
            assert srch <= even


def test_clt_search_against_a_continuous_optimum(golden_dir):
    # the hand-worked unit's per-head constants (b_N / z^2 and b_D / z^2 at
    # eps1 = eps2 = 1/20, from the golden fractions) give the budget at any
    # split in closed form; a continuous minimiser over (f, g) bounds the grid
    # search from below, and the grid point next to the continuous optimum
    # from above
    from scipy.optimize import minimize
    from scipy.stats import norm
    q, k, v, idx, base, n_t, want, prm = _clt_unit(golden_dir)
    eps, delta = prm["eps"], prm["delta"]
    cn = max(want[("bN", h)][0] / want[("bN", h)][1] for h in range(2)) / 400.0
    cd = max(want[("bD", h)][0] / want[("bD", h)][1] for h in range(2)) / 400.0

    def b_at(x):
        f, g = x
        zn, zd = norm.ppf(1 - g * delta / 2), norm.ppf(1 - (1 - g) * delta / 2)
        return max(zn ** 2 * cn / (f * eps / 2) ** 2, zd ** 2 * cd / ((1 - f) * eps / 2) ** 2)

    res = minimize(b_at, x0=[0.5, 0.5], method="Nelder-Mead", bounds=[(0.05, 0.95), (0.05, 0.95)],
                   options={"xatol": 1e-9, "fatol": 1e-9, "maxiter": 4000})
    _, det = budget.clt_budget_search(q, k, v, idx, base, math.log(2.0), eps, delta, n_t)
    assert det["b_real"] >= res.fun * (1 - 1e-9)
    near = min((abs(f - res.x[0]) + abs(g - res.x[1]), f, g) for f in budget.GRID for g in budget.GRID)
    assert det["b_real"] <= b_at((near[1], near[2])) * (1 + 1e-9)
    assert det["b_real"] == pytest.approx(b_at((det["f"], det["g"])), rel=1e-9)


def test_clt_search_corner_when_the_denominator_is_exact():
    # every key row zero: every logit 0, every weight 1, so the denominator's
    # sample variance is 0 and b_D = 0 at every split; the search then gives
    # the numerator the largest grid share of eps and delta (19/20 each), and
    # b is the lemma at eps1 = 0.95 eps / 2, delta1 = 0.95 delta
    r = np.random.default_rng(3)
    L, d, G = 4000, 4, 2
    k = np.zeros((L, d))
    v = 1.0 + 0.2 * r.standard_normal((L, d))
    q = r.standard_normal((G, d))
    idx = np.arange(100)
    base = np.arange(100, 164)
    n_t = L - 100
    eps, delta = 0.2, 0.05
    b, det = budget.clt_budget_search(q, k, v, idx, base, 0.3, eps, delta, n_t)
    assert det["f"] == 0.95 and det["g"] == 0.95
    n_hat = v[idx].sum(axis=0) + (n_t / 64) * v[base].sum(axis=0)
    tr = float(v[base].var(axis=0, ddof=1).sum())
    want = (norm_ppf(1 - 0.95 * delta / 2) * n_t * math.sqrt(tr) / (0.95 * eps / 2 * np.linalg.norm(n_hat))) ** 2
    assert det["b_real"] == pytest.approx(want, rel=1e-9)
    assert b == min(max(math.ceil(want), 64), n_t)


def norm_ppf(p):
    from scipy.stats import norm
    return float(norm.ppf(p))
