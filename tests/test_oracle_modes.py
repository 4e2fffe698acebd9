"""Pins for oracle.modes against torch's attention, algebraic identities the
pages fix, and statistics of the sampling estimator."""
import math

import numpy as np
import pytest
import torch

from oracle import modes, rng, select, stats


def _sdpa(q, k, v, scale):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), scale=scale)[0, 0].numpy()


def _unit(seed, G=4, L=512, d=16, sigma=1.0, n_hh=4):
    r = np.random.default_rng(seed)
    mu_q = r.standard_normal((G, d))
    mu_k = r.standard_normal(d)
    k = mu_k + sigma * r.standard_normal((L, d))
    u = mu_q.sum(0) / np.linalg.norm(mu_q.sum(0))
    k[r.choice(L, n_hh, replace=False)] += 4 * u
    v = r.standard_normal((L, d))
    q_ctx = mu_q[:, None, :] + r.standard_normal((G, L, d))
    q = mu_q + r.standard_normal((G, d))
    return q, k, v, q_ctx


def _setup(seed, **kw):
    q, k, v, q_ctx = _unit(seed, **kw)
    L, d = k.shape
    s = 1 / math.sqrt(d)
    st = stats.prefill_stats(q_ctx, k, v, s, "f32")
    return q, k, v, st, s


def test_dense_matches_torch_sdpa():
    q, k, v, st, s = _setup(0)
    np.testing.assert_allclose(modes.dense(q, k, v, s), _sdpa(q, k, v, s), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("mode", ["drop", "resa", "proxy", "sample"])
def test_full_budget_is_dense(mode):
    q, k, v, st, s = _setup(1)
    L = k.shape[0]
    idx = np.arange(L)
    out = modes.run_mode(mode, q, k, v, idx, st, s, pos=np.zeros(0, dtype=np.int64))
    np.testing.assert_allclose(out, _sdpa(q, k, v, s), rtol=1e-12, atol=1e-13)


def test_drop_is_attention_on_the_subset():
    q, k, v, st, s = _setup(2)
    idx = np.sort(np.random.default_rng(0).choice(k.shape[0], 77, replace=False))
    np.testing.assert_allclose(modes.drop(q, k, v, idx, s), _sdpa(q, k[idx], v[idx], s),
                               rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("lam", [1.0, 0.5, 0.1])
def test_resa_delta_merge_equals_merged_logit_softmax(lam):
    q, k, v, st, s = _setup(3)
    for nsel in (0, 1, 40, 300, 511):
        idx = np.sort(np.random.default_rng(nsel).choice(k.shape[0], nsel, replace=False))
        a = modes.resa(q, k, v, idx, st, s, lam)
        b = modes.resa_merged_logits(q, k, v, idx, st, s, lam)
        np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)


def test_resa_exact_when_keys_identical():
    # K_j = mu_K for all j: delta_i = (q_i - mu_Q)(K - mu_K)^T = 0, so the
    # prior logits plus bias equal the true ones and RESA is dense attention
    q, k, v, q_ctx = _unit(4)
    k[:] = k[0]
    s = 0.25
    st = stats.prefill_stats(q_ctx, k, v, s, "f32")
    idx = select.index_set(k.shape[0], 16, 32, [5, 9])
    np.testing.assert_allclose(modes.resa(q, k, v, idx, st, s), _sdpa(q, k, v, s),
                               rtol=1e-12, atol=1e-13)


def test_resa_lambda_zero_is_drop_and_empty_set_is_prior():
    q, k, v, st, s = _setup(5)
    idx = select.index_set(k.shape[0], 16, 32, [4, 11, 20])
    np.testing.assert_allclose(modes.resa(q, k, v, idx, st, s, 0.0), modes.drop(q, k, v, idx, s),
                               rtol=1e-13, atol=1e-14)
    # nothing read exactly: the output is the prior alone, O_Est (the bias
    # shifts every prior logit equally and cancels in the softmax)
    empty = np.zeros(0, dtype=np.int64)
    np.testing.assert_allclose(modes.resa(q, k, v, empty, st, s), st["o_est"], rtol=1e-12, atol=1e-13)


def test_resa_bias_aligns_prior_with_true_logits():
    # the bias c = s (q - mu_Q) . mu_K makes the prior logit exact at every
    # key equal to mu_K; check against the true logit directly
    q, k, v, st, s = _setup(6)
    kj = st["mu_k"]
    prior = s * st["mu_q"] @ kj + s * (q - st["mu_q"]) @ st["mu_k"]
    np.testing.assert_allclose(prior, s * q @ kj, rtol=1e-13)


def test_proxy_exact_for_one_token_tail():
    q, k, v, st, s = _setup(7, L=64)
    idx = select.index_set(64, 16, 47, [])          # tail = {16}
    assert select.tail_set(64, idx).tolist() == [16]
    np.testing.assert_allclose(modes.proxy(q, k, v, idx, st, s), _sdpa(q, k, v, s),
                               rtol=1e-12, atol=1e-13)


def test_proxy_exact_for_identical_tail_keys_and_values():
    q, k, v, st0, s = _setup(8)
    idx = select.index_set(k.shape[0], 16, 32, [3, 17])
    tail = select.tail_set(k.shape[0], idx)
    k[tail] = k[tail[0]]
    v[tail] = v[tail[0]]
    q_ctx = np.random.default_rng(0).standard_normal((4, k.shape[0], k.shape[1]))
    st = stats.prefill_stats(q_ctx, k, v, s, "f32")
    np.testing.assert_allclose(modes.proxy(q, k, v, idx, st, s), _sdpa(q, k, v, s),
                               rtol=1e-12, atol=1e-13)


def test_proxy_tail_means_from_totals_equal_direct_means():
    q, k, v, st, s = _setup(9)
    idx = select.index_set(k.shape[0], 16, 32, [6, 8])
    tail = select.tail_set(k.shape[0], idx)
    # the proxy with totals-minus-selected must equal a proxy built from the
    # tail rows directly
    kbar = k[tail].mean(0)
    vbar = v[tail].mean(0)
    z = s * q @ kbar + math.log(len(tail))
    lg = np.concatenate([s * q @ k[idx].T, z[:, None]], 1)
    w = np.exp(lg - lg.max(1, keepdims=True))
    want = (w[:, :-1] @ v[idx] + w[:, -1:] * vbar) / w.sum(1, keepdims=True)
    np.testing.assert_allclose(modes.proxy(q, k, v, idx, st, s), want, rtol=1e-12, atol=1e-13)


def test_sample_exact_for_identical_tail_tokens():
    q, k, v, st, s = _setup(10)
    idx = select.index_set(k.shape[0], 16, 32, [2, 9, 30])
    tail = select.tail_set(k.shape[0], idx)
    k[tail] = k[tail[3]]
    v[tail] = v[tail[3]]
    pos = rng.sample_positions(77, 0, 0, 0, tail, 13)
    np.testing.assert_allclose(modes.sample(q, k, v, idx, pos, s), _sdpa(q, k, v, s),
                               rtol=1e-12, atol=1e-13)


def test_sample_estimator_unbiased_over_seeds():
    # N_hat and D_hat (not their ratio) are unbiased for the tail sums
    q, k, v, st, s = _setup(11, L=384)
    L = k.shape[0]
    idx = select.index_set(L, 16, 32, [4, 10])
    tail = select.tail_set(L, idx)
    shift = (s * q @ k.T).max(1)
    e_t = np.exp(s * q @ k[tail].T - shift[:, None])
    e_i = np.exp(s * q @ k[idx].T - shift[:, None])
    n_true = e_i @ v[idx] + e_t @ v[tail]
    d_true = e_i.sum(1) + e_t.sum(1)
    b, n_seeds = 16, 4000
    ns, ds = [], []
    for seed in range(n_seeds):
        pos = rng.sample_positions(seed, 0, 0, 0, tail, b)
        nh, dh = modes.sample_num_den(q, k, v, idx, pos, s, shift)
        ns.append(nh)
        ds.append(dh)
    ns, ds = np.array(ns), np.array(ds)
    se_n = ns.std(0) / math.sqrt(n_seeds)
    se_d = ds.std(0) / math.sqrt(n_seeds)
    assert np.all(np.abs(ns.mean(0) - n_true) <= 5 * se_n + 1e-12)
    assert np.all(np.abs(ds.mean(0) - d_true) <= 5 * se_d + 1e-12)


def _loop_unit(mode, q, k, v, idx, st, s, pos):
    """Plain-loop restatement on tiny inputs (brute force, no numpy algebra)."""
    G, d = q.shape
    L = k.shape[0]
    I = set(int(i) for i in idx)
    T = [j for j in range(L) if j not in I]
    dot = lambda a, b: sum(a[i] * b[i] for i in range(d))
    out = []
    for h in range(G):
        terms = []  # (log-weight, value row)
        for j in sorted(I):
            terms.append((s * dot(q[h], k[j]), list(v[j])))
        if T and mode == "proxy":
            kb = [sum(k[j][i] for j in T) / len(T) for i in range(d)]
            vb = [sum(v[j][i] for j in T) / len(T) for i in range(d)]
            terms.append((s * dot(q[h], kb) + math.log(len(T)), vb))
        if T and mode == "sample":
            for j in pos:
                terms.append((s * dot(q[h], k[j]) + math.log(len(T) / len(pos)), list(v[j])))
        if T and mode == "resa":
            c = s * dot([q[h][i] - st["mu_q"][h][i] for i in range(d)], st["mu_k"])
            for j in T:
                terms.append((s * dot(st["mu_q"][h], k[j]) + c, list(v[j])))
        m = max(t[0] for t in terms)
        ws = [math.exp(t[0] - m) for t in terms]
        out.append([sum(w * t[1][i] for w, t in zip(ws, terms)) / sum(ws) for i in range(d)])
    return np.array(out)


@pytest.mark.parametrize("mode", ["drop", "resa", "proxy", "sample"])
def test_modes_against_plain_loops(mode):
    q, k, v, q_ctx = _unit(12, G=2, L=96, d=4)
    s = 0.5
    st = stats.prefill_stats(q_ctx, k, v, s, "f32")
    blocks, idx, tail = select.select_unit(q, st["blk_mean"], 96, 16, 16, 2)
    pos = rng.sample_positions(5, 0, 0, 3, tail, 9)
    got = modes.run_mode(mode, q, k, v, idx, st, s, pos=pos)
    np.testing.assert_allclose(got, _loop_unit(mode, q, k, v, idx, st, s, pos), rtol=1e-11, atol=1e-12)


def test_empty_exact_set():
    q, k, v, st, s = _setup(13)
    empty = np.zeros(0, dtype=np.int64)
    assert np.array_equal(modes.drop(q, k, v, empty, s), np.zeros((q.shape[0], v.shape[1])))
    assert np.array_equal(modes.resa(q, k, v, empty, st, s, 0.0), np.zeros((q.shape[0], v.shape[1])))
    # the proxy alone is the tail-mean value (one token carries all weight)
    np.testing.assert_allclose(modes.proxy(q, k, v, empty, st, s), np.tile(v.mean(0), (q.shape[0], 1)),
                               rtol=1e-12, atol=1e-13)


def test_sample_per_head_reductions():
    # every head drawing the same positions gives the group estimator; one
    # head alone is the one-head estimator; heads with different draws differ
    from oracle import modes as M
    r = np.random.default_rng(17)
    G, d, L = 3, 8, 256
    q = r.standard_normal((G, d))
    k = r.standard_normal((L, d))
    v = r.standard_normal((L, d))
    idx = np.arange(0, 40)
    tail = np.arange(40, L)
    pos = r.choice(tail, 24)
    same = M.sample_per_head(q, k, v, idx, [pos] * G, 0.3)
    assert np.allclose(same, M.sample(q, k, v, idx, pos, 0.3), rtol=0, atol=1e-14)
    per = [r.choice(tail, n) for n in (8, 16, 32)]
    got = M.sample_per_head(q, k, v, idx, per, 0.3)
    for h in range(G):
        assert np.allclose(got[h], M.sample(q[h:h + 1], k, v, idx, per[h], 0.3)[0], rtol=0, atol=1e-14)
    assert not np.allclose(got, M.sample(q, k, v, idx, per[0], 0.3))
