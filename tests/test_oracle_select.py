"""Pins for oracle.select: brute-force ranking, ties, known block order."""
import itertools

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
