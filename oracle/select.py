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

Parity pins (tests/test_oracle_select.py): brute force over all subsets on
tiny inputs, sorting with Python's own sort, all-equal scores, planted blocks
whose rank is known, scores against exact rational arithmetic, ties between
identical and permuted summaries.
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


def select_unit(q, blk_mean, L, sink, local, k_blocks):
    """Full selection of one unit: (chosen blocks ascending, I, T)."""
    cand = candidate_blocks(L, sink, local)
    sc = block_scores(q, blk_mean, cand)
    blocks = top_blocks(sc, cand, k_blocks)
    idx = index_set(L, sink, local, blocks)
    return blocks, idx, tail_set(L, idx)
