"""The oracle's pins catch plausible mistakes: each test plants one mistake in
an oracle function (on the CPU, by replacing it for the duration of the
test) and checks that at least one of the pins written for that function
fails.  A pin set that passed a planted mistake would not be pinning it."""
import math

import numpy as np
import pytest

import oracle.modes as modes
import oracle.numerics as numerics
import oracle.select as select
import oracle.stats as stats
import test_oracle_modes as pin_modes
import test_oracle_numerics as pin_num
import test_oracle_select as pin_sel
import test_oracle_stats as pin_stats


def _some_pin_fails(pins):
    """True when at least one of the (function, kwargs) pins raises an
    AssertionError."""
    for fn, kw in pins:
        try:
            fn(**kw)
        except AssertionError:
            return True
    return False


# ---- planted mistakes ---------------------------------------------------------

def _resa_without_bias(q, k, v, idx, st, scale, lam=1.0, _orig=modes.resa):
    # the bias c = s (q - mu_Q) . mu_K dropped (mu_K enters resa only there)
    return _orig(q, k, v, idx, dict(st, mu_k=0.0 * st["mu_k"]), scale, lam)


def _resa_lambda_on_alpha_only(q, k, v, idx, st, scale, lam=1.0):
    # lambda applied to alpha alone, not to the prior mass inside Z'
    n_t = k.shape[0] - len(idx)
    if n_t == 0 or len(idx) == 0:
        return modes.drop(q, k, v, idx, scale) if n_t == 0 else st["o_est"].copy()
    kI, vI = k[idx], v[idx]
    c = scale * ((q - st["mu_q"]) @ st["mu_k"])
    l_i = scale * (q @ kI.T)
    p_i = scale * (st["mu_q"] @ kI.T) + c[:, None]
    log_z = st["log_z0"] + c
    m = np.maximum(np.maximum(log_z, l_i.max(1)), p_i.max(1))[:, None]
    z = np.exp(log_z[:, None] - m)
    e_p, e_l = np.exp(p_i - m), np.exp(l_i - m)
    z_new = np.maximum(z[:, 0] - e_p.sum(1), 0.0) + e_l.sum(1)
    alpha = lam * z[:, 0] / z_new
    return alpha[:, None] * st["o_est"] + (e_l / z_new[:, None] - alpha[:, None] * e_p / z) @ vI


def _proxy_without_log_n(q, k, v, idx, st, scale):
    n_t = k.shape[0] - len(idx)
    if n_t == 0:
        return modes.drop(q, k, v, idx, scale)
    kbar = (st["sum_k"] - k[idx].sum(0)) / n_t
    vbar = (st["sum_v"] - v[idx].sum(0)) / n_t
    z = scale * (q @ kbar)                                        # + ln n_T missing
    logits = np.concatenate([scale * (q @ k[idx].T), z[:, None]], axis=1)
    return modes._softmax_weighted(logits, np.concatenate([v[idx], vbar[None]], axis=0))


def _sample_without_weight(q, k, v, idx, pos, scale):
    n_t = k.shape[0] - len(idx)
    if n_t == 0 or len(pos) == 0:
        return modes.drop(q, k, v, idx, scale)
    logits = np.concatenate([scale * (q @ k[idx].T), scale * (q @ k[pos].T)], axis=1)  # no ln(n_T / b)
    return modes._softmax_weighted(logits, np.concatenate([v[idx], v[pos]], axis=0))


def _sample_num_den_without_weight(q, k, v, idx, pos, scale, shift):
    e_i = np.exp(scale * (q @ k[idx].T) - shift[:, None])
    e_s = np.exp(scale * (q @ k[pos].T) - shift[:, None])      # the n_T / b factor missing
    return e_i @ v[idx] + e_s @ v[pos], e_i.sum(1) + e_s.sum(1)


def _top_blocks_high_index_first(scores, cand, k):
    k = min(int(k), len(cand))
    order = np.lexsort((-cand, -scores))                          # ties to the HIGHER index
    return np.sort(cand[order[:k]])


def _round_to_bf16_7_bits(x):
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = x != 0
    _, e = np.frexp(x[nz])
    sp = np.maximum(e - 7, -133)                                  # one bit short
    out[nz] = np.ldexp(np.rint(np.ldexp(x[nz], -sp)), sp)
    return out


def _block_means_over_15(k, kv_dtype):
    L, d = k.shape
    nb = L // 16
    return numerics.round_to(k[: nb * 16].reshape(nb, 16, d).sum(axis=1) / 15.0, kv_dtype)


# ---- the checks -----------------------------------------------------------------

MODE_PINS = [
    (pin_modes.test_full_budget_is_dense, {"mode": m}) for m in ("drop", "resa", "proxy", "sample")
] + [
    (pin_modes.test_resa_delta_merge_equals_merged_logit_softmax, {"lam": lam}) for lam in (1.0, 0.5)
] + [
    (pin_modes.test_resa_exact_when_keys_identical, {}),
    (pin_modes.test_resa_lambda_zero_is_drop_and_empty_set_is_prior, {}),
    (pin_modes.test_proxy_exact_for_one_token_tail, {}),
    (pin_modes.test_proxy_exact_for_identical_tail_keys_and_values, {}),
    (pin_modes.test_proxy_tail_means_from_totals_equal_direct_means, {}),
    (pin_modes.test_sample_exact_for_identical_tail_tokens, {}),
    (pin_modes.test_sample_estimator_unbiased_over_seeds, {}),
]


@pytest.mark.parametrize("name,attr,mutant", [
    ("dropped RESA bias", "resa", _resa_without_bias),
    ("lambda on alpha only", "resa", _resa_lambda_on_alpha_only),
    ("proxy without + ln n_T", "proxy", _proxy_without_log_n),
    ("sample without n_T / b", "sample", _sample_without_weight),
    ("estimator without n_T / b", "sample_num_den", _sample_num_den_without_weight),
])
def test_mode_mistakes_fail_a_pin(name, attr, mutant, monkeypatch):
    monkeypatch.setattr(modes, attr, mutant)
    assert _some_pin_fails(MODE_PINS), name


def test_reversed_tie_break_fails_a_pin(monkeypatch):
    monkeypatch.setattr(select, "top_blocks", _top_blocks_high_index_first)
    pins = [(pin_sel.test_all_equal_scores_take_lowest_indices, {}),
            (pin_sel.test_identical_summaries_tie_anywhere, {}),
            (pin_sel.test_permuted_summaries_tie_under_a_constant_query, {})]
    pins += [(pin_sel.test_top_blocks_brute_force, {"seed": s}) for s in range(3)]
    assert _some_pin_fails(pins)


def test_wrong_bf16_spacing_fails_a_pin(monkeypatch):
    monkeypatch.setattr(numerics, "round_to_bf16", _round_to_bf16_7_bits)
    monkeypatch.setattr(pin_num, "round_to_bf16", _round_to_bf16_7_bits)
    pins = [(pin_num.test_bf16_matches_torch_cast_on_fp32_values, {}),
            (pin_num.test_bf16_ties_and_single_rounding, {})]
    assert _some_pin_fails(pins)


def test_wrong_block_mean_divisor_fails_a_pin(monkeypatch):
    monkeypatch.setattr(stats, "block_means", _block_means_over_15)
    monkeypatch.setattr(pin_stats, "block_means", _block_means_over_15)
    pins = [(pin_stats.test_block_means_against_torch_cast, {}),
            (pin_stats.test_constant_keys_closed_form, {})]
    assert _some_pin_fails(pins)


def test_unmutated_oracle_passes_every_pin_used_here():
    """The same pins pass on the oracle as written (so the checks above fail
    because of the planted mistakes, not on their own)."""
    pins = MODE_PINS + [(pin_sel.test_all_equal_scores_take_lowest_indices, {}),
                        (pin_num.test_bf16_ties_and_single_rounding, {}),
                        (pin_stats.test_block_means_against_torch_cast, {})]
    for fn, kw in pins:
        fn(**kw)


def _mix64_wrong_shift(z, _M=(1 << 64) - 1):
    z &= _M
    z = ((z ^ (z >> 31)) * 0xBF58476D1CE4E5B9) & _M               # 30 -> 31
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M
    return z ^ (z >> 31)


def _z_one_sided(delta):
    from scipy.stats import norm
    return float(norm.ppf(1.0 - delta))                           # one-sided quantile


def _grown_stats_prefix_prior(st0, k, v, scale, kv_dtype, _orig=stats.grown_stats):
    # O_Est and log_z0 left at their prefill-end values (appended tokens ignored)
    g = _orig(st0, k, v, scale, kv_dtype)
    return dict(g, o_est=st0["o_est"], log_z0=st0["log_z0"])


def test_rng_mixer_mistake_fails_a_pin(monkeypatch, golden_dir):
    import oracle.rng as rng
    import test_oracle_rng as pin_rng
    monkeypatch.setattr(rng, "mix64", _mix64_wrong_shift)
    assert _some_pin_fails([(pin_rng.test_splitmix64_reference_outputs, {"golden_dir": golden_dir}),
                            (pin_rng.test_mixer_is_a_bijection_on_samples, {})])


def test_budget_quantile_mistake_fails_a_pin(monkeypatch, golden_dir):
    import oracle.budget as budget
    import test_oracle_budget as pin_budget
    monkeypatch.setattr(budget, "z_two_sided", _z_one_sided)
    assert _some_pin_fails([(pin_budget.test_lemma_worked_example, {"golden_dir": golden_dir}),
                            (pin_budget.test_quantile_textbook_values, {})])


def test_grown_prior_mistake_fails_a_pin(monkeypatch):
    monkeypatch.setattr(stats, "grown_stats", _grown_stats_prefix_prior)
    monkeypatch.setattr(pin_stats, "grown_stats", _grown_stats_prefix_prior)
    assert _some_pin_fails([(pin_stats.test_grown_stats_follow_the_token_recurrence, {}),
                            (pin_stats.test_grown_stats_constant_keys_closed_form, {})])


def _clt_budget_variant(eps_div=4.0, delta_div=2.0, scale_up=True, ddof=1, reduce_heads=max):
    """oracle.budget.clt_budget restated with one step changeable, to plant a
    mistake in the budget's composition."""
    import oracle.budget as budget

    def f(q, k, v, idx, base_pos, scale, eps, delta, n_t):
        b0 = len(base_pos)
        if n_t == 0 or b0 < 2:
            return 0, {}
        e1, d1 = eps / eps_div, delta / delta_div
        l_i, l_s = scale * (q @ k[idx].T), scale * (q @ k[base_pos].T)
        m = np.maximum(l_i.max(axis=1), l_s.max(axis=1))
        e_i, e_s = np.exp(l_i - m[:, None]), np.exp(l_s - m[:, None])
        w = n_t / b0 if scale_up else 1.0
        n_hat = e_i @ v[idx] + w * (e_s @ v[base_pos])
        d_hat = e_i.sum(axis=1) + w * e_s.sum(axis=1)
        det = {"b_N": [], "b_D": []}
        per_head = []
        for h in range(q.shape[0]):
            r = e_s[h][:, None] * v[base_pos]
            b_n = budget.lemma_budget(n_t, float(r.var(axis=0, ddof=ddof).sum()),
                                      e1 * float(np.linalg.norm(n_hat[h])), d1)
            b_d = budget.lemma_budget(n_t, float(e_s[h].var(ddof=ddof)), e1 * float(d_hat[h]), d1)
            det["b_N"].append(b_n)
            det["b_D"].append(b_d)
            per_head.append(max(b_n, b_d))
        best = reduce_heads(per_head)
        b = int(min(max(math.ceil(best) if math.isfinite(best) else n_t, b0), n_t))
        return b, det
    return f


CLT_MISTAKES = {
    "eps split in two, not four": dict(eps_div=2.0),
    "delta not split": dict(delta_div=1.0),
    "no n_T / b0 scale-up of the base sample": dict(scale_up=False),
    "biased (ddof 0) spreads": dict(ddof=0),
    "min over the query heads": dict(reduce_heads=min),
}


@pytest.mark.parametrize("name", list(CLT_MISTAKES))
def test_clt_budget_mistake_fails_a_pin(monkeypatch, golden_dir, name):
    import oracle.budget as budget
    import test_oracle_budget as pin_budget
    pins = [(pin_budget.test_clt_budget_hand_worked_unit, {"golden_dir": golden_dir}),
            (pin_budget.test_clt_budget_clamps_to_the_tail, {"golden_dir": golden_dir})]
    monkeypatch.setattr(budget, "clt_budget", _clt_budget_variant())
    for fn, kw in pins:                       # the restatement itself passes
        fn(**kw)
    monkeypatch.setattr(budget, "clt_budget", _clt_budget_variant(**CLT_MISTAKES[name]))
    assert _some_pin_fails(pins)


def _max_heads_as_sum(q, blk_mean, cand, _orig=select.block_scores):
    return _orig(q, blk_mean, cand)                                  # sum over heads, not max


def _max_heads_as_mean_query(q, blk_mean, cand, _orig=select.block_scores):
    return _orig(np.asarray(q).max(axis=0, keepdims=True), blk_mean, cand)   # max of the query, not of the scores


def _quest_upper_only(q, blk_min, blk_max, cand):
    q = np.asarray(q, dtype=np.float64)
    return np.array([math.fsum((q * np.asarray(blk_max)[c]).ravel()) for c in cand])   # min branch dropped


def _quest_swapped(q, blk_min, blk_max, cand):
    q = np.asarray(q, dtype=np.float64)
    return np.array([math.fsum(np.minimum(q * np.asarray(blk_min)[c], q * np.asarray(blk_max)[c]).ravel())
                     for c in cand])                                 # lower bound instead of the upper


def _minmax_shifted(k):
    L, d = k.shape
    nb = L // 16
    b = k[1: nb * 16 + 1] if L >= nb * 16 + 1 else k[: nb * 16]     # block boundaries off by one token
    b = b.reshape(-1, 16, d)
    return b.min(axis=1), b.max(axis=1)


SELECTOR_MISTAKES = {
    "max over heads taken as the sum": ("block_scores_max_heads", _max_heads_as_sum),
    "max over heads of the query, not the scores": ("block_scores_max_heads", _max_heads_as_mean_query),
    "quest without the min branch": ("block_scores_quest", _quest_upper_only),
    "quest taking the lower bound": ("block_scores_quest", _quest_swapped),
}


@pytest.mark.parametrize("name", list(SELECTOR_MISTAKES))
def test_selector_variant_mistake_fails_a_pin(monkeypatch, name):
    attr, fn = SELECTOR_MISTAKES[name]
    monkeypatch.setattr(select, attr, fn)
    monkeypatch.setattr(pin_sel.S, attr, fn)
    pins = [(pin_sel.test_max_heads_scores_exact_rational, {"seed": s}) for s in range(3)]
    pins += [(pin_sel.test_max_heads_planted_single_head_winner, {})]
    pins += [(pin_sel.test_quest_scores_exact_rational, {"seed": s}) for s in range(3)]
    pins += [(pin_sel.test_quest_score_bounds_every_token_of_its_block, {})]
    assert _some_pin_fails(pins)


def test_block_minmax_mistake_fails_a_pin(monkeypatch):
    monkeypatch.setattr(stats, "block_minmax", _minmax_shifted)
    assert _some_pin_fails([(pin_stats.test_block_minmax_against_loops_and_torch, {})])


def _search_variant(eps_half=True, delta_g=1.0):
    import oracle.budget as budget

    def f_(q, k, v, idx, base_pos, scale, eps, delta, n_t):
        b0 = len(base_pos)
        n_hat, d_hat, e_s, r = budget._estimates(q, k, v, idx, base_pos, scale, n_t)
        G = q.shape[0]
        tr = [float(r[h].var(axis=0, ddof=1).sum()) for h in range(G)]
        vd = [float(e_s[h].var(ddof=1)) for h in range(G)]
        best = (math.inf, None, None)
        for f in budget.GRID:
            e1 = f * eps / 2.0 if eps_half else f * eps
            e2 = (1.0 - f) * eps / 2.0 if eps_half else (1.0 - f) * eps
            for g in budget.GRID:
                d1, d2 = g * delta * delta_g, (1.0 - g) * delta * delta_g
                b = 0.0
                for h in range(G):
                    b = max(b, budget.lemma_budget(n_t, tr[h], e1 * float(np.linalg.norm(n_hat[h])), d1),
                            budget.lemma_budget(n_t, vd[h], e2 * float(d_hat[h]), d2))
                if b < best[0]:
                    best = (b, f, g)
        return budget._clamp(best[0], b0, n_t), {"b_real": best[0], "f": best[1], "g": best[2]}
    return f_


def _hoeffding_variant(union=True, use_range=True):
    import oracle.budget as budget

    def f_(q, k, v, idx, base_pos, scale, eps, delta, n_t):
        b0 = len(base_pos)
        n_hat, d_hat, e_s, r = budget._estimates(q, k, v, idx, base_pos, scale, n_t)
        G, d = q.shape[0], v.shape[1]
        e1 = e2 = eps / 4.0
        d1 = d2 = delta / 2.0
        det = {"b_N": [], "b_D": []}
        best = 0.0
        for h in range(G):
            if use_range:
                rn2 = float(((r[h].max(axis=0) - r[h].min(axis=0)) ** 2).max())
                rd2 = float((e_s[h].max() - e_s[h].min()) ** 2)
            else:                                                   # spread by the standard deviation
                rn2 = float(r[h].var(axis=0, ddof=1).max())
                rd2 = float(e_s[h].var(ddof=1))
            tn, td = e1 * float(np.linalg.norm(n_hat[h])), e2 * float(d_hat[h])
            dd = d if union else 1
            b_n = dd * n_t ** 2 * math.log(2.0 * dd / d1) * rn2 / (2.0 * tn ** 2)
            b_d = n_t ** 2 * math.log(2.0 / d2) * rd2 / (2.0 * td ** 2)
            det["b_N"].append(b_n)
            det["b_D"].append(b_d)
            best = max(best, b_n, b_d)
        return budget._clamp(best, b0, n_t), det
    return f_


BUDGET_RULE_MISTAKES = {
    "search: eps split not halved": ("clt_budget_search", _search_variant(eps_half=False)),
    "search: delta halved again": ("clt_budget_search", _search_variant(delta_g=0.5)),
    "hoeffding: no union bound over coordinates": ("hoeffding_budget", _hoeffding_variant(union=False)),
    "hoeffding: spread instead of range": ("hoeffding_budget", _hoeffding_variant(use_range=False)),
}


@pytest.mark.parametrize("name", list(BUDGET_RULE_MISTAKES))
def test_budget_rule_mistake_fails_a_pin(monkeypatch, golden_dir, name):
    import oracle.budget as budget
    import test_oracle_budget as pin_budget
    pins = [(pin_budget.test_hoeffding_hand_worked_unit, {"golden_dir": golden_dir}),
            (pin_budget.test_clt_search_against_a_continuous_optimum, {"golden_dir": golden_dir}),
            (pin_budget.test_clt_search_corner_when_the_denominator_is_exact, {})]
    attr, fn = BUDGET_RULE_MISTAKES[name]
    monkeypatch.setattr(budget, attr, _search_variant() if attr == "clt_budget_search" else _hoeffding_variant())
    for p_, kw in pins:                      # the restatements themselves pass
        p_(**kw)
    monkeypatch.setattr(budget, attr, fn)
    assert _some_pin_fails(pins)


def _multi_proxy_without_log_n(q, k, v, read, assign, cs, scale):
    import oracle.openattn as OA
    cs2 = dict(cs)
    out_logits, out_vals = [scale * (q @ k[read].T)], [v[read]]
    for c in range(len(cs["n"])):
        mr = read[assign[read] == c] if len(read) else read
        n_un = int(cs["n"][c]) - len(mr)
        if n_un <= 0:
            continue
        kb = (cs["sum_k"][c] - k[mr].sum(axis=0)) / n_un
        vb = (cs["sum_v"][c] - v[mr].sum(axis=0)) / n_un
        out_logits.append((scale * (q @ kb))[:, None])                  # + ln n' missing
        out_vals.append(vb[None, :])
    lg = np.concatenate(out_logits, axis=1)
    w = np.exp(lg - lg.max(axis=1, keepdims=True))
    return (w @ np.concatenate(out_vals, axis=0)) / w.sum(axis=1, keepdims=True)


def _kmeans_frozen(y, n_clusters=64, rounds=10):
    L = len(y)
    cent = y[(np.arange(n_clusters) * L) // n_clusters].copy()          # never moved
    d2 = ((y[:, None, :] - cent[None, :, :]) ** 2).sum(axis=2)
    return np.argmin(d2, axis=1), cent


def _errors_without_variance(q, cs, scale):
    n = cs["n"].astype(np.float64)
    live = n > 0
    mean = np.zeros_like(cs["sum_k"])
    mean[live] = cs["sum_k"][live] / n[live, None]
    mu = scale * (q @ mean.T)
    return np.where(live[None, :], n[None, :] * np.exp(mu - mu.max(axis=1, keepdims=True)), 0).sum(axis=0)


def _scores_without_scale(qq, code, sig):
    from oracle.numerics import round_to_f32
    return round_to_f32((code @ qq).astype(np.float64))


OPENATTN_MISTAKES = {
    "proxy logit without ln n": ("multi_proxy", _multi_proxy_without_log_n),
    "k-means centroids never updated": ("kmeans", _kmeans_frozen),
    "weight error without the variance": ("cluster_errors", _errors_without_variance),
    "QGS score without the token scale": ("qgs_scores", _scores_without_scale),
}


@pytest.mark.parametrize("name", list(OPENATTN_MISTAKES))
def test_openattn_mistake_fails_a_pin(monkeypatch, name):
    import oracle.openattn as OA
    import test_oracle_openattn as pin_oa
    attr, fn = OPENATTN_MISTAKES[name]
    monkeypatch.setattr(OA, attr, fn)
    pins = [(getattr(pin_oa, t), {}) for t in dir(pin_oa) if t.startswith("test_")]
    assert _some_pin_fails(pins)


def test_openattn_uncapped_split_fails_a_pin(monkeypatch):
    import oracle.openattn as OA
    import test_oracle_openattn as pin_oa
    orig = OA.errorgate
    monkeypatch.setattr(OA, "errorgate", lambda err, n, budget: orig(err, np.full(len(n), 10 ** 9), budget))
    assert _some_pin_fails([(pin_oa.test_errorgate_caps_and_totals, {})])
