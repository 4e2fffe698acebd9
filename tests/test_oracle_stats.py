"""Pins for oracle.stats: closed forms and an independent attention routine."""
import math

import numpy as np
import torch

from oracle.numerics import round_to_bf16
from oracle.stats import block_means, grown_stats, prefill_stats


def _sdpa(q, k, v, scale):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), scale=scale)[0, 0].numpy()


def test_constant_keys_closed_form():
    rng = np.random.default_rng(0)
    G, L, d = 3, 96, 8
    kappa = round_to_bf16(rng.standard_normal(d))
    k = np.tile(kappa, (L, 1))
    v = rng.standard_normal((L, d))
    mu = rng.standard_normal((G, d))
    noise = rng.standard_normal((G, L // 2, d))
    q_ctx = mu[:, None, :] + np.concatenate([noise, -noise], axis=1)  # mean exactly mu
    s = 1 / math.sqrt(d)
    st = prefill_stats(q_ctx, k, v, s, "bf16")
    np.testing.assert_allclose(st["mu_q"], mu, rtol=0, atol=1e-13)
    np.testing.assert_array_equal(st["mu_k"], kappa)
    np.testing.assert_allclose(st["sum_k"], L * kappa, rtol=1e-15)
    np.testing.assert_allclose(st["log_z0"], math.log(L) + s * (mu @ kappa), rtol=0, atol=1e-12)
    np.testing.assert_allclose(st["o_est"], np.tile(v.mean(0), (G, 1)), atol=1e-13)
    np.testing.assert_array_equal(st["blk_mean"], np.tile(kappa, (L // 16, 1)))
    assert st["kbar_absmax"] == np.abs(kappa).max()


def test_o_est_is_attention_of_the_typical_query():
    rng = np.random.default_rng(1)
    G, L, d = 4, 256, 16
    q_ctx = rng.standard_normal((G, L, d)) + rng.standard_normal((G, 1, d))
    k = rng.standard_normal((L, d)) * 2
    v = rng.standard_normal((L, d))
    s = 0.3
    st = prefill_stats(q_ctx, k, v, s, "f32")
    mu = q_ctx.mean(axis=1)
    np.testing.assert_allclose(st["o_est"], _sdpa(mu, k, v, s), rtol=1e-12, atol=1e-12)
    lse = torch.logsumexp(torch.from_numpy(s * mu @ k.T), dim=1).numpy()
    np.testing.assert_allclose(st["log_z0"], lse, rtol=1e-14)


def test_block_means_against_torch_cast():
    # blocks of 16 small integers times 2^-6: the fp64 mean is exactly an
    # fp32 value, so torch's fp32 -> bf16 cast is an independent reference
    rng = np.random.default_rng(2)
    L, d = 16 * 50, 32
    k = rng.integers(-3000, 3000, size=(L, d)).astype(np.float64) * 2.0 ** -6
    means32 = (k.reshape(-1, 16, d).sum(1) / 16).astype(np.float32)
    assert np.array_equal(means32.astype(np.float64), k.reshape(-1, 16, d).mean(1))
    want = torch.from_numpy(means32).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(block_means(k, "bf16"), want)
    np.testing.assert_array_equal(block_means(k, "f32"), means32.astype(np.float64))


def test_grown_stats_follow_the_token_recurrence():
    """Statistics of a cache grown past prefill end: the definition over all
    L' tokens equals folding the appended tokens in one at a time from the
    prefill-end values (log-sum-exp of the normaliser, mass-weighted mix of
    O_Est, running totals), the arithmetic an incremental update performs."""
    rng = np.random.default_rng(3)
    G, L0, n, d = 2, 64, 37, 16
    s = 0.25
    q_ctx = rng.standard_normal((G, L0, d)) + rng.standard_normal((G, 1, d))
    k = rng.standard_normal((L0 + n, d)) * 1.5
    v = rng.standard_normal((L0 + n, d))
    st0 = prefill_stats(q_ctx, k[:L0], v[:L0], s, "f32")
    lz, o = st0["log_z0"].copy(), st0["o_est"].copy()
    sk, sv = st0["sum_k"].copy(), st0["sum_v"].copy()
    for j in range(L0, L0 + n):
        p = s * (st0["mu_q"] @ k[j])
        lz_new = np.logaddexp(lz, p)
        o = np.exp(lz - lz_new)[:, None] * o + np.exp(p - lz_new)[:, None] * v[j][None, :]
        lz = lz_new
        sk, sv = sk + k[j], sv + v[j]
    g = grown_stats(st0, k, v, s, "f32")
    np.testing.assert_allclose(g["log_z0"], lz, rtol=1e-13)
    np.testing.assert_allclose(g["o_est"], o, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(g["sum_k"], sk, rtol=1e-13, atol=1e-12)
    np.testing.assert_allclose(g["sum_v"], sv, rtol=1e-13, atol=1e-12)
    # the typical query and key stay the prefill-end ones
    assert g["mu_q"] is st0["mu_q"] and g["mu_k"] is st0["mu_k"]
    # complete blocks only: (64 + 37) // 16 = 6 means, the first 4 as at prefill
    assert g["blk_mean"].shape == (6, d)
    np.testing.assert_array_equal(g["blk_mean"][:4], st0["blk_mean"])


def test_grown_stats_constant_keys_closed_form():
    """Constant keys kappa over a length that is not a whole number of blocks:
    log_z0 = ln L' + s mu_Q . kappa and O_Est = the mean of all L' values."""
    rng = np.random.default_rng(4)
    G, L0, n, d = 3, 48, 21, 8
    kappa = round_to_bf16(rng.standard_normal(d))
    k = np.tile(kappa, (L0 + n, 1))
    v = rng.standard_normal((L0 + n, d))
    q_ctx = rng.standard_normal((G, L0, d))
    s = 1 / math.sqrt(d)
    st0 = prefill_stats(q_ctx, k[:L0], v[:L0], s, "bf16")
    g = grown_stats(st0, k, v, s, "bf16")
    Lg = L0 + n
    np.testing.assert_allclose(g["log_z0"], math.log(Lg) + s * (st0["mu_q"] @ kappa), rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["o_est"], np.tile(v.mean(0), (G, 1)), atol=1e-13)
    np.testing.assert_allclose(g["sum_k"], Lg * kappa, rtol=1e-15)
    np.testing.assert_array_equal(g["blk_mean"], np.tile(kappa, (Lg // 16, 1)))


def test_block_minmax_against_loops_and_torch():
    from oracle import stats as ostats
    # elementwise min / max over each complete 16-token block, the partial
    # last block left out: Python loops and torch's amin / amax over the
    # reshaped cache agree exactly (values of the cache, no rounding)
    import torch
    rng = np.random.default_rng(21)
    L, d = 16 * 9 + 5, 6
    k = rng.standard_normal((L, d)).astype(np.float32).astype(np.float64)
    mn, mx = ostats.block_minmax(k)
    assert mn.shape == (9, d) and mx.shape == (9, d)
    for c in range(9):
        for e in range(d):
            col = [k[16 * c + j, e] for j in range(16)]
            assert mn[c, e] == min(col) and mx[c, e] == max(col)
    t = torch.from_numpy(k[: 16 * 9]).reshape(9, 16, d)
    assert np.array_equal(mn, t.amin(dim=1).numpy()) and np.array_equal(mx, t.amax(dim=1).numpy())
