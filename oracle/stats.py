"""Prefill-end statistics of one unit (sequence b, KV head g).

Follows RESA, Method, key design 1 ("Prior Estimator"):
  * the typical query mu_Q and typical key mu_K are means of the historical
    queries / keys; here mu_Q[h] is the mean over the L context queries of
    query head h, and mu_K the mean of the L cached keys of the KV head;
  * the prior logit row mu_Q K^T / sqrt(d) does not depend on the decode
    query, so it is computed once at prefill end: its softmax-weighted sum of
    V is O_Est and its exponential sum is the normaliser (stored as
    log_z0 = ln sum_j exp(s * mu_Q . K_j), without the query-dependent bias);
    this is the "one extra query appended at prefill end, L -> L+1".

Also the totals the count-aware proxy needs (OpenAttention, stage 04: tail
sums are totals minus the selected part), and the 16-token block means the
block selector ranks (Quest/ArkVale-style page summaries named on the RESA
page's related work), rounded once to the cache dtype, and each block's
elementwise key minimum and maximum (Quest's per-page bounds, the summaries
of the "quest" block score).

Decode grows the cache after prefill end (grown_stats): the statistics then
describe all cached tokens while the typical query and key stay the ones of
prefill end.  Reading: the RESA page fixes mu_Q and mu_K at prefill end and
defines O_Est and the normaliser as the typical query's attention over the
cache, which its tail estimate removes the read set from; so O_Est, log_z0
and the totals cover every cached token, and mu_K (also the centre the block
sketch is built around) does not move.

Parity pins (tests/test_oracle_stats.py): closed forms for constant keys /
queries (log_z0 = ln L + s mu_Q.kappa, O_Est = mean V), O_Est against torch's
scaled_dot_product_attention with query mu_Q, block means against torch's
bf16 cast where the mean is an fp32 value; block minima and maxima against
Python loops and torch's amin / amax; grown statistics against a
token-by-token log-sum-exp recurrence from the prefill-end values and
against constant-key closed forms at lengths that are not whole blocks.
"""
import numpy as np

from .numerics import round_to

BLOCK = 16


def block_means(k, kv_dtype):
    """k [L, d] float64 -> [L//16, d]: mean of each complete 16-token block,
    computed in fp64 and rounded once to the cache dtype (nearest, ties to
    even); a partial last block has no mean."""
    L, d = k.shape
    nb = L // BLOCK
    return round_to(k[: nb * BLOCK].reshape(nb, BLOCK, d).mean(axis=1), kv_dtype)


def block_minmax(k):
    """k [L, d] -> (min, max) [L//16, d]: the elementwise minimum and maximum
    of the keys of each complete 16-token block (Quest's per-page key
    bounds); values of the cache, so no rounding."""
    L, d = k.shape
    nb = L // BLOCK
    blocks = k[: nb * BLOCK].reshape(nb, BLOCK, d)
    return blocks.min(axis=1), blocks.max(axis=1)


def prefill_stats(q_ctx, k, v, scale, kv_dtype):
    """q_ctx [G, L, d], k [L, d], v [L, d] (float64 holding the cache values).

    Returns a dict with
      mu_q [G, d], o_est [G, d], log_z0 [G],            (per query head)
      mu_k [d], sum_k [d], sum_v [d],                    (per KV head)
      blk_mean [L/16, d] (cache dtype values), kbar_absmax (max |blk_mean|).
    """
    G, L, d = q_ctx.shape
    mu_q = q_ctx.mean(axis=1)
    sum_k = k.sum(axis=0)
    sum_v = v.sum(axis=0)
    mu_k = sum_k / L
    p0 = scale * (mu_q @ k.T)                  # prior logits of the typical query [G, L]
    m = p0.max(axis=1, keepdims=True)
    w = np.exp(p0 - m)
    a = w.sum(axis=1)
    log_z0 = np.log(a) + m[:, 0]
    o_est = (w @ v) / a[:, None]
    bm = block_means(k, kv_dtype)
    mn, mx = block_minmax(k)
    return {
        "mu_q": mu_q, "o_est": o_est, "log_z0": log_z0,
        "mu_k": mu_k, "sum_k": sum_k, "sum_v": sum_v,
        "blk_mean": bm, "kbar_absmax": float(np.abs(bm).max()),
        "blk_min": mn, "blk_max": mx,
    }


def grown_stats(st0, k, v, scale, kv_dtype):
    """Statistics of a cache that holds L' = len(k) tokens after growing past
    prefill end, with the typical query and key of prefill end (st0["mu_q"],
    st0["mu_k"]): O_Est and log_z0 of mu_Q over all L' keys, the totals of
    all L' keys and values, and the means of the complete blocks."""
    mu_q = st0["mu_q"]
    p0 = scale * (mu_q @ k.T)                  # prior logits [G, L']
    m = p0.max(axis=1, keepdims=True)
    w = np.exp(p0 - m)
    a = w.sum(axis=1)
    bm = block_means(k, kv_dtype)
    mn, mx = block_minmax(k)
    return {
        "blk_min": mn, "blk_max": mx,
        "mu_q": mu_q, "o_est": (w @ v) / a[:, None], "log_z0": np.log(a) + m[:, 0],
        "mu_k": st0["mu_k"], "sum_k": k.sum(axis=0), "sum_v": v.sum(axis=0),
        "blk_mean": bm, "kbar_absmax": float(np.abs(bm).max()) if len(bm) else 0.0,
    }
