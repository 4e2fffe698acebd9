"""Pins for oracle.select: brute-force ranking, ties, known block order,
exact scores."""
import itertools
from fractions import Fraction

import numpy as np
import pytest

from oracle import select as S


def _brute_force(scores, cand, k):
    # c is chosen iff fewer than k candidates beat it, where c' beats c when
    # its score is larger or equal with a smaller block index
    chosen = []
    for i, c in enumerate(cand):
        beaten_by = sum(1 for j, c2 in enumerate(cand)
                        if scores[j] > scores[i] or (scores[j] == scores[i] and c2 < c))
        if beaten_by < k:
            chosen.append(c)
    return sorted(chosen)


@pytest.mark.parametrize("seed", range(20))
def test_top_blocks_brute_force(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 12))
    cand = np.sort(rng.choice(40, size=n, replace=False)).astype(np.int64)
    scores = rng.integers(-3, 4, size=n).astype(np.float64)   # many ties
    for k in range(0, n + 2):
        got = S.top_blocks(scores, cand, k).tolist()
        assert got == _brute_force(scores, cand, k)
        # and Python's own sort with the same key
        py = sorted(sorted(zip(cand.tolist(), scores.tolist()), key=lambda t: (-t[1], t[0]))[:k])
        assert got == [c for c, _ in py]


def test_all_equal_scores_take_lowest_indices():
    rng = np.random.default_rng(3)
    d = 8
    row = rng.standard_normal(d)
    blk = np.tile(row, (40, 1))
    q = rng.standard_normal((4, d))
    blocks, idx, tail = S.select_unit(q, blk, 640, 16, 32, 5)
    assert blocks.tolist() == [1, 2, 3, 4, 5]


def test_planted_blocks_rank_known():
    rng = np.random.default_rng(4)
    d, nb = 16, 64
    q = rng.standard_normal((2, d))
    u = q.sum(0) / np.linalg.norm(q.sum(0))
    base = rng.standard_normal((nb, d))
    base -= np.outer(base @ u, u)                     # orthogonal to the group query
    t = rng.permutation(nb).astype(np.float64)        # distinct strengths
    blk = base + np.outer(t, u)
    cand = S.candidate_blocks(nb * 16, 0, 0)
    got = S.top_blocks(S.block_scores(q, blk, cand), cand, 7)
    assert got.tolist() == sorted(np.argsort(-t)[:7].tolist())


def test_candidate_ranges_and_index_sets():
    assert S.candidate_blocks(2048, 16, 32).tolist() == list(range(1, 126))
    assert S.candidate_blocks(64, 16, 47).tolist() == []          # only partial blocks
    assert S.candidate_blocks(64, 20, 10).tolist() == [2]         # 20..54: block 2 = 32..48
    assert S.candidate_blocks(64, 40, 40).tolist() == []          # sink and window overlap
    idx = S.index_set(2048, 16, 32, [3, 7, 100])
    assert len(idx) == 16 + 32 + 48 and idx.tolist() == sorted(set(idx.tolist()))
    tail = S.tail_set(2048, idx)
    assert len(tail) + len(idx) == 2048 and not set(tail) & set(idx)
    assert S.index_set(64, 40, 40, []).tolist() == list(range(64))
    # partial blocks beside the sink / window stay in the tail
    idx2 = S.index_set(64, 20, 10, [2])
    assert S.tail_set(64, idx2).tolist() == [20, 21, 22, 23, 24, 25, 26, 27, 28, 29, 30, 31,
                                              48, 49, 50, 51, 52, 53]


def _f32(a):
    return np.asarray(a, dtype=np.float32).astype(np.float64)


@pytest.mark.parametrize("seed", range(6))
def test_scores_are_the_exact_value_rounded_once(seed):
    # rational arithmetic is exact; float(Fraction) rounds once to nearest
    rng = np.random.default_rng(100 + seed)
    G, d, nb = 3, 24, 9
    q = _f32(rng.standard_normal((G, d)) * 2.0 ** rng.integers(-20, 20, (G, d)))
    blk = _f32(rng.standard_normal((nb, d)) * 2.0 ** rng.integers(-20, 20, (nb, d)))
    cand = np.arange(nb)
    got = S.block_scores(q, blk, cand)
    for i in range(nb):
        exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(q.ravel(), np.tile(blk[i], G)))
        assert got[i] == float(exact)


def test_identical_summaries_tie_anywhere():
    # the same summary row at many positions: equal scores, lowest indices win
    # (two heads, d = 64, 182 rows: a shape where a plain fp64 matrix product
    # rounds identical rows differently depending on their position)
    rng = np.random.default_rng(7)
    G, d, nb = 2, 64, 182
    q = _f32(rng.standard_normal((G, d)))
    rows = _f32(rng.standard_normal((5, d)))
    pick = rng.integers(0, 5, nb)
    blk = rows[pick]
    cand = np.arange(nb)
    sc = S.block_scores(q, blk, cand)
    for r in range(5):
        assert len(set(sc[pick == r].tolist())) == 1
    best = max(range(5), key=lambda r: sc[pick == r][0])
    want = np.flatnonzero(pick == best)[:3]
    assert S.top_blocks(sc, cand, 3).tolist() == want.tolist()


def test_permuted_summaries_tie_under_a_constant_query():
    # q_he = const for all e: a permutation of a row leaves the exact score
    # unchanged, so every permutation ties with the original
    rng = np.random.default_rng(8)
    d = 64
    q = _f32(np.full((2, d), 0.3))
    row = _f32(rng.standard_normal(d) * 2.0 ** rng.integers(-30, 30, d))
    blk = np.stack([row[rng.permutation(d)] for _ in range(20)])
    sc = S.block_scores(q, blk, np.arange(20))
    assert len(set(sc.tolist())) == 1
    assert S.top_blocks(sc, np.arange(20), 4).tolist() == [0, 1, 2, 3]
