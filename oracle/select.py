"""Exactly-read index set I of one unit: sink + local window + top blocks.

Follows vAttention, Method, overall framework: the deterministic set I_f is
the attention sink (first tokens), the local window (latest tokens) and the
top-scoring tokens of an approximate top-k.  The top-k here ranks 16-token
blocks by their mean key (the block-level selection of Quest / ArkVale that
the RESA page wraps), one index set per KV head because the group's query
heads share the K/V reads.

Readings where the pages are silent:
  * candidate blocks are those that do not overlap the sink or the window;
  * score_c = sum_{h in group} q_h . kbar_c (the 1/sqrt(d) factor is positive
    and common, so it does not change the ranking and is left out);
  * ties go to the lower block index: rank by (score desc, index asc);
  * the decision is taken in fp64 on the exact score rounded once: the real
    number sum_h sum_e q_he kbar_ce (q and kbar are bf16 / fp32 values, so
    each product is exact in fp64) correctly rounded by fsum.  Equal real
    scores therefore compare equal whatever the order of the terms, and two
    blocks with identical summaries always tie.

Two other block scores, the alternatives the RESA page's related work (the
page-level top-k selectors it builds on: Quest, ArkVale) and the GQA
reading of "per-head top-k" leave open:
  * "mean_max": score_c = max_{h in group} q_h . kbar_c, the group's
    strongest head decides (each head's exact dot product rounded once; the
    max of the rounded values is the rounded max, rounding being monotone);
  * "quest": per block the elementwise minimum and maximum of its keys,
    score_c = sum_h sum_e max(q_he min_ce, q_he max_ce), for each head an
    upper bound of q_h . K_j over the block's tokens (Quest's criticality
    bound), summed over the group like the default score; each term is one
    of two exact products, summed exactly and rounded once.
Both rank by (score desc, index asc) like the default "mean_sum".

Parity pins (tests/test_oracle_select.py): brute force over all subsets on
tiny inputs, sorting with Python's own sort, all-equal scores, planted blocks
whose rank is known, scores against exact rational arithmetic, ties between
identical and permuted summaries; for the two alternatives exact rational
arithmetic on small integers, the single-head reduction to the default
score (mean_max), the upper-bound property and its equality on constant
blocks (quest), planted winners.
"""
import math

import numpy as np

BLOCK = 16


def candidate_blocks(L, sink, local):
    """Blocks c with [16c, 16c+16) disjoint from [0, sink) and [L-local, L)."""
    lo = -(-sink // BLOCK)
    hi = max(L - local, 0) // BLOCK
    return np.arange(lo, max(hi, lo), dtype=np.int64)


def block_scores(q, blk_mean, cand):
    """q [G, d], blk_mean [nb, d] (bf16 / fp32 values) -> score of each
    candidate block: sum over heads and dims of q_he * kbar_ce, every product
    exact in fp64, summed exactly and rounded once (math.fsum)."""
    q = np.asarray(q, dtype=np.float64)
    blk_mean = np.asarray(blk_mean, dtype=np.float64)
    out = np.empty(len(cand), dtype=np.float64)
    for i, c in enumerate(cand):
        out[i] = math.fsum((q * blk_mean[c]).ravel())
    return out


def block_scores_max_heads(q, blk_mean, cand):
    """max over heads of the exact q_h . kbar_c (each rounded once by fsum)."""
    q = np.asarray(q, dtype=np.float64)
    blk_mean = np.asarray(blk_mean, dtype=np.float64)
    out = np.empty(len(cand), dtype=np.float64)
    for i, c in enumerate(cand):
        out[i] = max(math.fsum(q[h] * blk_mean[c]) for h in range(q.shape[0]))
    return out


def block_scores_quest(q, blk_min, blk_max, cand):
    """sum over heads and dims of max(q_he min_ce, q_he max_ce), every term an
    exact fp64 product, summed exactly and rounded once (math.fsum)."""
    q = np.asarray(q, dtype=np.float64)
    blk_min = np.asarray(blk_min, dtype=np.float64)
    blk_max = np.asarray(blk_max, dtype=np.float64)
    out = np.empty(len(cand), dtype=np.float64)
    for i, c in enumerate(cand):
        out[i] = math.fsum(np.maximum(q * blk_min[c], q * blk_max[c]).ravel())
    return out


SCORES = ("mean_sum", "mean_max", "quest")


def scores_for(score, q, st, cand):
    """Block scores of the candidates by the named score; st holds blk_mean
    (and blk_min, blk_max for "quest")."""
    if score == "mean_sum":
        return block_scores(q, st["blk_mean"], cand)
    if score == "mean_max":
        return block_scores_max_heads(q, st["blk_mean"], cand)
    if score == "quest":
        return block_scores_quest(q, st["blk_min"], st["blk_max"], cand)
    raise ValueError(score)


def top_blocks(scores, cand, k):
    """The k best candidates by (score desc, block index asc), returned in
    ascending block order."""
    k = min(int(k), len(cand))
    order = np.lexsort((cand, -scores))        # last key is the primary key
    return np.sort(cand[order[:k]])


def index_set(L, sink, local, blocks):
    """Sorted token positions read exactly: [0,sink) u [L-local,L) u blocks."""
    mask = np.zeros(L, dtype=bool)
    mask[: min(sink, L)] = True
    mask[max(L - local, 0):] = True
    for c in blocks:
        mask[BLOCK * c: BLOCK * c + BLOCK] = True
    return np.flatnonzero(mask)


def tail_set(L, idx):
    """Sorted positions not read exactly (the residual / tail T)."""
    mask = np.ones(L, dtype=bool)
    mask[idx] = False
    return np.flatnonzero(mask)


def select_unit(q, blk_mean, L, sink, local, k_blocks, score="mean_sum", st=None):
    """Full selection of one unit: (chosen blocks ascending, I, T).  score
    other than "mean_sum" takes the summaries from st."""
    cand = candidate_blocks(L, sink, local)
    sc = block_scores(q, blk_mean, cand) if score == "mean_sum" else scores_for(score, q, st, cand)
    blocks = top_blocks(sc, cand, k_blocks)
    idx = index_set(L, sink, local, blocks)
    return blocks, idx, tail_set(L, idx)
