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


# ---- the two alternative block scores (max over heads; Quest min/max bounds) ----

def _frac_rows(a):
    return [[Fraction(x) for x in row] for row in np.asarray(a).tolist()]


@pytest.mark.parametrize("seed", range(6))
def test_max_heads_scores_exact_rational(seed):
    # dyadic small values: every score is an exact rational; the oracle's
    # scores equal max_h sum_e q_he kbar_ce computed in Fractions, and its
    # top-k equals brute force over those exact scores
    rng = np.random.default_rng(100 + seed)
    G, d, nb = 3, 8, 40
    q = rng.integers(-6, 7, size=(G, d)) / 8.0
    blk = rng.integers(-5, 6, size=(nb, d)) / 4.0
    cand = np.arange(2, nb - 3, dtype=np.int64)
    got = S.block_scores_max_heads(q, blk, cand)
    qf, bf = _frac_rows(q), _frac_rows(blk)
    exact = [max(sum(a * b for a, b in zip(qf[h], bf[c])) for h in range(G)) for c in cand]
    assert [Fraction(x) for x in got] == exact
    for k in (0, 1, 5, len(cand)):
        assert S.top_blocks(got, cand, k).tolist() == _brute_force(exact, cand.tolist(), k)


def test_max_heads_with_one_head_is_the_default_score():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 16)).astype(np.float32).astype(np.float64)
    blk = rng.standard_normal((50, 16)).astype(np.float32).astype(np.float64)
    cand = np.arange(50, dtype=np.int64)
    assert np.array_equal(S.block_scores_max_heads(q, blk, cand), S.block_scores(q, blk, cand))


def test_max_heads_planted_single_head_winner():
    # block 5 matches head 0 strongly and the other heads weakly against it;
    # block 9 matches every head moderately: the group sum prefers 9, the
    # max over heads prefers 5
    d = 4
    q = np.array([[4.0, 0, 0, 0], [0, 1.0, 0, 0], [0, 0, 1.0, 0]])
    blk = np.zeros((16, d))
    blk[5] = [2.0, -1.0, -1.0, 0]          # head scores 8, -1, -1: sum 6, max 8
    blk[9] = [1.0, 2.0, 2.0, 0]            # head scores 4, 2, 2: sum 8, max 4
    cand = np.arange(16, dtype=np.int64)
    assert S.top_blocks(S.block_scores(q, blk, cand), cand, 1).tolist() == [9]
    assert S.top_blocks(S.block_scores_max_heads(q, blk, cand), cand, 1).tolist() == [5]


@pytest.mark.parametrize("seed", range(6))
def test_quest_scores_exact_rational(seed):
    rng = np.random.default_rng(200 + seed)
    G, d, L = 2, 6, 16 * 12
    q = rng.integers(-6, 7, size=(G, d)) / 4.0
    k = rng.integers(-9, 10, size=(L, d)) / 8.0
    mn, mx = _block_minmax_loops(k)
    cand = np.arange(1, 11, dtype=np.int64)
    got = S.block_scores_quest(q, mn, mx, cand)
    qf, mnf, mxf = _frac_rows(q), _frac_rows(mn), _frac_rows(mx)
    exact = [sum(max(qf[h][e] * mnf[c][e], qf[h][e] * mxf[c][e]) for h in range(G) for e in range(d))
             for c in cand]
    assert [Fraction(x) for x in got] == exact
    for kk in (1, 3, len(cand)):
        assert S.top_blocks(got, cand, kk).tolist() == _brute_force(exact, cand.tolist(), kk)


def _block_minmax_loops(k):
    nb = k.shape[0] // 16
    mn = np.array([[min(k[16 * c + j, e] for j in range(16)) for e in range(k.shape[1])] for c in range(nb)])
    mx = np.array([[max(k[16 * c + j, e] for j in range(16)) for e in range(k.shape[1])] for c in range(nb)])
    return mn, mx


def test_quest_score_bounds_every_token_of_its_block():
    # per head, sum_e max(q_e min_e, q_e max_e) >= q . K_j for every token j of
    # the block; rounding is monotone, so the rounded bound is >= the rounded
    # largest logit (exact rational logits, rounded once by float()), with
    # equality when the block's keys are all one row; the group score is the
    # exact sum of the heads' exact bounds, rounded once
    rng = np.random.default_rng(11)
    G, d, L = 3, 8, 16 * 20
    q = rng.standard_normal((G, d)).astype(np.float32).astype(np.float64)
    k = rng.standard_normal((L, d)).astype(np.float32).astype(np.float64)
    k[16 * 7: 16 * 8] = k[16 * 7]                      # block 7: sixteen copies of one key
    mn, mx = _block_minmax_loops(k)
    cand = np.arange(20, dtype=np.int64)
    exact_group = [Fraction(0)] * len(cand)
    for h in range(G):
        bound = S.block_scores_quest(q[h:h + 1], mn, mx, cand)
        for c in cand:
            top = max(_exact_dot(q[h], k[16 * c + j]) for j in range(16))
            assert bound[c] >= float(top)
            if c == 7:
                assert bound[c] == float(top)
            exact_group[c] += sum(max(Fraction(a) * Fraction(lo), Fraction(a) * Fraction(hi))
                                  for a, lo, hi in zip(q[h].tolist(), mn[c].tolist(), mx[c].tolist()))
    assert S.block_scores_quest(q, mn, mx, cand).tolist() == [float(x) for x in exact_group]


def _exact_dot(a, b):
    return sum(Fraction(x) * Fraction(y) for x, y in zip(a.tolist(), b.tolist()))


def test_select_unit_with_alternative_scores():
    rng = np.random.default_rng(5)
    G, d, L = 4, 16, 16 * 64
    q = rng.standard_normal((G, d))
    k = rng.standard_normal((L, d))
    from oracle import stats
    st = stats.prefill_stats(rng.standard_normal((G, L, d)), k, rng.standard_normal((L, d)), 0.25, "f32")
    for score in S.SCORES:
        blocks, idx, tail = S.select_unit(q, st["blk_mean"], L, 16, 32, 6, score=score, st=st)
        cand = S.candidate_blocks(L, 16, 32)
        want = S.top_blocks(S.scores_for(score, q, st, cand), cand, 6)
        assert blocks.tolist() == want.tolist()
        assert len(idx) == 16 + 32 + 6 * 16 and len(idx) + len(tail) == L
