"""Pins for oracle.openattn (the OpenAttention multi-proxy pipeline): the
query basis, k-means, the ErrorGate split, the QGS scores and the
multi-proxy output, each against something other than itself."""
import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import modes, openattn as OA
from oracle.numerics import round_to_f32


def test_query_basis_spans_a_planted_subspace():
    # queries confined to a random 5-dimensional subspace of R^12: the top 5
    # eigenvectors span it (projector equal), the rest carry no mass, and the
    # columns are orthonormal eigenvectors of the second moment
    r = np.random.default_rng(0)
    d, G, L = 12, 2, 400
    a = np.linalg.qr(r.standard_normal((d, 5)))[0]
    q_ctx = (r.standard_normal((G, L, 5)) * np.array([5, 4, 3, 2, 1.0])) @ a.T
    u, w = OA.query_basis(q_ctx, 5)
    assert np.allclose(u @ u.T, a @ a.T, atol=1e-10)
    assert np.allclose(w[5:], 0.0, atol=1e-10) and np.all(np.diff(w) <= 1e-12)
    m = q_ctx.reshape(-1, d).T @ q_ctx.reshape(-1, d) / (G * L)
    assert np.allclose(m @ u, u * w[:5], atol=1e-9)
    assert np.allclose(u.T @ u, np.eye(5), atol=1e-12)


def test_kmeans_recovers_separated_blobs():
    # four well-separated blobs laid out in position order, so that the
    # starts floor(c L / C) fall one in each: the clusters are the blobs
    r = np.random.default_rng(1)
    centres = np.array([[10.0, 0], [0, 10.0], [-10.0, 0], [0, -10.0]])
    y = np.concatenate([c + 0.5 * r.standard_normal((50, 2)) for c in centres])
    a, cent = OA.kmeans(y, n_clusters=4, rounds=10)
    assert a.tolist() == sum([[c] * 50 for c in range(4)], [])
    for c in range(4):
        assert np.allclose(cent[c], y[a == c].mean(axis=0))


def test_kmeans_ends_at_its_fixed_point():
    # after the final assignment every point is nearest to its own centroid
    # (computed here by brute force over all centroids) and every non-empty
    # centroid of the last round is its members' mean
    r = np.random.default_rng(2)
    y = r.standard_normal((300, 3))
    a, cent = OA.kmeans(y, n_clusters=7, rounds=30)
    for j in range(len(y)):
        dist = [float(((y[j] - cent[c]) ** 2).sum()) for c in range(7)]
        assert a[j] == dist.index(min(dist))
    for c in range(7):
        if (a == c).any():
            assert np.allclose(cent[c], y[a == c].mean(axis=0), atol=1e-12)


def test_cluster_stats_closed_forms():
    r = np.random.default_rng(3)
    k = r.standard_normal((90, 4))
    v = r.standard_normal((90, 4))
    a = np.arange(90) % 3
    cs = OA.cluster_stats(k, v, a, 5)
    assert cs["n"].tolist() == [30, 30, 30, 0, 0]
    for c in range(3):
        assert np.allclose(cs["sum_k"][c], sum(k[j] for j in range(c, 90, 3)))
        assert np.allclose(cs["sum_v"][c], sum(v[j] for j in range(c, 90, 3)))
        assert np.allclose(cs["sum_k2"][c], sum(k[j] * k[j] for j in range(c, 90, 3)))
    assert not cs["sum_k"][3:].any()


def test_errorgate_hand_worked_split():
    # errors 3 : 1 : 0 (rescaled to 2^30 : 2^30/3 : 0), 10 tokens:
    # floor(10 * 3/4) = 7 (remainder 2^31 of W = 4 2^30 / 3 ...), worked with
    # integers below; the cluster without error gets nothing while others have room
    w0, w1 = 2 ** 30, int(np.rint(2 ** 30 / 3))
    W = w0 + w1
    q = OA.errorgate([3.0, 1.0, 0.0], [100, 100, 100], 10)
    q0, q1 = 10 * w0 // W, 10 * w1 // W
    left = 10 - q0 - q1
    rem = {0: 10 * w0 % W, 1: 10 * w1 % W, 2: 0}
    order = sorted(rem, key=lambda c: (-rem[c], c))
    want = {0: q0, 1: q1, 2: 0}
    for c in order[:left]:
        want[c] += 1
    assert q.tolist() == [want[0], want[1], want[2]]
    assert q.sum() == 10 and q[2] == 0


def test_errorgate_caps_and_totals():
    # a cluster asking for more than it holds is capped and its share goes to
    # the others; the total is min(budget, tokens); no error at all spreads
    # the budget by index
    q = OA.errorgate([5.0, 1.0, 1.0], [2, 50, 50], 20)
    assert q.sum() == 20 and q[0] == 2 and q[1] + q[2] == 18 and abs(int(q[1]) - int(q[2])) <= 1
    assert OA.errorgate([1.0, 1.0], [3, 4], 50).tolist() == [3, 4]
    assert OA.errorgate([0.0, 0.0, 0.0], [5, 5, 5], 4).tolist() == [2, 1, 1]


def test_cluster_errors_zero_for_exact_clusters():
    # a cluster whose keys are all equal has zero variance: no weight error
    r = np.random.default_rng(4)
    d = 6
    k = np.concatenate([np.tile(r.standard_normal(d), (40, 1)), r.standard_normal((40, d))])
    v = r.standard_normal((80, d))
    a = np.repeat([0, 1], 40)
    cs = OA.cluster_stats(k, v, a, 2)
    err = OA.cluster_errors(r.standard_normal((3, d)), cs, 0.4)
    assert err[1] > 0.0 and err[0] <= 1e-12 * err[1]      # zero up to the rounding of E[k^2] - E[k]^2


def test_qgs_scores_exact_integers():
    r = np.random.default_rng(5)
    d, L = 8, 40
    u = round_to_f32(np.linalg.qr(r.standard_normal((d, 4)))[0])
    k = round_to_f32(r.standard_normal((L, d)))
    code, sig = OA.qgs_codes(k, u)
    # the codes reproduce z within half a scale step, with the largest at 127
    z = np.array([[float(sum(Fraction(x) * Fraction(y) for x, y in zip(k[j], u[:, i]))) for i in range(4)]
                  for j in range(L)])
    assert np.all(np.abs(z - sig[:, None] * code) <= sig[:, None] / 2 + 1e-12)
    assert np.all(np.abs(code).max(axis=1) == 127)
    qq = OA.qgs_query(r.standard_normal((3, d)), u)
    s = OA.qgs_scores(qq, code, sig)
    for j in range(L):
        exact = Fraction(float(sig[j])) * sum(int(a) * int(b) for a, b in zip(qq, code[j]))
        assert s[j] == float(np.float32(float(exact)))
    assert np.abs(qq).max() == 32767


def test_select_tokens_brute_force():
    r = np.random.default_rng(6)
    L = 60
    scores = r.integers(-3, 4, size=L).astype(np.float64)      # many ties
    a = r.integers(0, 4, size=L)
    qb = [2, 0, 5, 1]
    got = OA.select_tokens(scores, a, qb)
    want = []
    for c in range(4):
        mem = [j for j in range(L) if a[j] == c]
        mem.sort(key=lambda j: (-scores[j], j))
        want += mem[: qb[c]]
    assert got.tolist() == sorted(want)


def _unit(seed, L=256, d=8, G=2):
    r = np.random.default_rng(seed)
    return r.standard_normal((G, d)), r.standard_normal((L, d)), r.standard_normal((L, d))


def test_multi_proxy_full_read_is_dense():
    q, k, v = _unit(7)
    a = np.arange(len(k)) % 5
    cs = OA.cluster_stats(k, v, a, 5)
    got = OA.multi_proxy(q, k, v, np.arange(len(k)), a, cs, 0.35)
    assert np.allclose(got, modes.dense(q, k, v, 0.35), atol=1e-12)


def test_multi_proxy_identical_keys_is_dense():
    # every cluster's keys identical: each proxy carries exactly its members'
    # mass and mean value, so the output is dense attention whatever is read
    r = np.random.default_rng(8)
    d, L = 6, 120
    rows = r.standard_normal((4, d))
    a = np.repeat(np.arange(4), 30)
    k = rows[a]
    v = r.standard_normal((L, d))
    q = r.standard_normal((3, d))
    cs = OA.cluster_stats(k, v, a, 4)
    read = np.array([0, 5, 31, 32, 90])
    got = OA.multi_proxy(q, k, v, read, a, cs, 0.5)
    assert np.allclose(got, modes.dense(q, k, v, 0.5), atol=1e-12)


def test_multi_proxy_one_cluster_nothing_read_is_the_single_proxy():
    q, k, v = _unit(9)
    a = np.zeros(len(k), dtype=np.int64)
    cs = OA.cluster_stats(k, v, a, 1)
    st = {"sum_k": k.sum(axis=0), "sum_v": v.sum(axis=0)}
    got = OA.multi_proxy(q, k, v, np.zeros(0, dtype=np.int64), a, cs, 0.3)
    assert np.allclose(got, modes.proxy(q, k, v, np.zeros(0, dtype=np.int64), st, 0.3), atol=1e-12)


def test_step_reads_the_budget():
    r = np.random.default_rng(10)
    G, d, L = 2, 16, 2048
    q_ctx = r.standard_normal((G, L, d))
    k = r.standard_normal((L, d))
    v = r.standard_normal((L, d))
    a, u32 = OA.qgc(q_ctx, k, 8)
    cs = OA.cluster_stats(k, v, a, 8)
    code, sig = OA.qgs_codes(k, u32, exact=False)
    read, qb, out = OA.step(r.standard_normal((G, d)), k, v, a, u32, cs, code, sig, 0.25, 40)
    assert len(read) == 40 and qb.sum() == 40 and len(set(read.tolist())) == 40
    assert np.all(np.bincount(a[read], minlength=8) == qb)
    assert np.all(np.isfinite(out))
