"""OpenAttention multi-proxy pipeline of one unit (KV head), fp64.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Follows "OpenAttention: One Percent Is Enough with Tail Proxies", method
overview stages 01-04:
  01 QGC: project the keys onto the top-16 eigenvectors of the query second
     moment and cluster them with k-means (C = 64); cache each cluster's
     count, mean key and diagonal variance (here as sums, so that the unread
     members' means follow by subtraction);
  02 ErrorGate: split a token budget E over the clusters in proportion to
     each cluster's estimated weight error;
  03 QGS: score every token with int8 codes of its key in the r = 32
     subspace of the same eigenvectors and read each cluster's top q_b;
  04 every cluster's unread members fold into one count-aware mean proxy
     (logit of the unread-mean key + ln of their count, value = their mean
     value), and one softmax runs over the exact tokens and the proxies.

Readings (the page gives the stages, not their formulas):
  * the second moment is over the unit's context queries (all G heads, all
    L positions), M = (1/(G L)) sum q q^T; its eigenvectors in order of
    decreasing eigenvalue, stored in fp32 (the basis a kernel reads: every
    product of a basis entry and a bf16 / fp32 value is then exact in fp64);
  * k-means (Lloyd) on the projected keys y_j = U16^T K_j: centroid c starts
    at y of position floor(c L / C); 10 rounds of (assign each key to the
    nearest centroid by squared distance, lowest index on ties; move each
    centroid to its members' mean, an empty one stays); the clusters are a
    last assignment to those centroids;
  * estimated weight error (ErrorGate): with the cached mean and diagonal
    variance a member's logit for head h is modelled as normal with mean
    mu = s q_h . Kbar_b and variance var = s^2 sum_e q_he^2 var_be; a proxy
    carrying n_b e^mu misses n_b e^mu (e^(var/2) - 1) of the expected mass
    n_b e^(mu + var/2) (the lognormal mean); per head that error is divided
    by the head's estimated total mass sum_b n_b e^(mu + var/2), and the
    cluster's error is the sum over the group's heads;
  * budget split: the errors are brought to integers w_b = rint(2^30 err_b /
    max err) (so that the integer allocation below is exact), q_b =
    min(n_b, floor(E w_b / W)), W = sum w, and the tokens left go one at a
    time to the clusters with room, by largest remainder (E w_b mod W) then
    lowest index, round after round;
  * QGS codes: z = U32^T K_j (each coordinate the exact sum rounded once),
    scale sigma_j = fl32(max |z| / 127), code = clamp(rint(z / sigma_j), +-127)
    (0 when sigma_j = 0); the group's projected query p = U32^T sum_h q_h
    (exact sums rounded once) is coded to 16 bits, sq = max |p| / 32767,
    qq = clamp(rint(p / sq), +-32767); a token's score is sigma_j (qq . code_j)
    (an exact integer dot times an fp32 scale, exact in fp64) rounded once to
    fp32; each cluster reads its top q_b tokens by (score desc, index asc);
  * no attention sink or local window: the budget E is the whole exact read
    (the page's pipeline has none).

Parity pins (tests/test_oracle_openattn.py): the basis against a planted
low-rank query set and the eigen-equation; k-means recovering planted
separated blobs and ending at its own fixed point; the allocation's
exactness (sums, caps, proportions on a hand-worked case, zero-variance
clusters); QGS scores against exact integer arithmetic; the output equal to
dense attention when every cluster is read in full or when every cluster's
keys are identical, and equal to the single count-aware proxy with one
cluster and nothing read.
"""
import math

import numpy as np

from .numerics import round_to_f32

C_CLUSTERS = 64
R_QGC = 16
R_QGS = 32
KMEANS_ROUNDS = 10


def query_basis(q_ctx, r):
    """q_ctx [G, L, d] -> the eigenvectors [d, r] of the r largest eigenvalues
    of M = (1/(G L)) sum q q^T (columns in decreasing eigenvalue order) and
    all eigenvalues, decreasing."""
    x = np.asarray(q_ctx, dtype=np.float64).reshape(-1, q_ctx.shape[-1])
    m = x.T @ x / len(x)
    w, vec = np.linalg.eigh(m)
    order = np.argsort(-w, kind="stable")
    return vec[:, order[:r]], w[order]


def kmeans(y, n_clusters=C_CLUSTERS, rounds=KMEANS_ROUNDS):
    """Lloyd's k-means of the rows of y [L, r] with the fixed start and round
    count above; returns (assignment [L] int64, centroids [C, r])."""
    L = len(y)
    cent = y[(np.arange(n_clusters) * L) // n_clusters].copy()

    def assign(c):
        a = np.empty(L, dtype=np.int64)
        for j0 in range(0, L, 4096):
            d2 = ((y[j0:j0 + 4096, None, :] - c[None, :, :]) ** 2).sum(axis=2)
            a[j0:j0 + 4096] = np.argmin(d2, axis=1)   # first minimum: lowest index
        return a

    for _ in range(rounds):
        a = assign(cent)
        for c in range(n_clusters):
            mem = a == c
            if mem.any():
                cent[c] = y[mem].mean(axis=0)
    return assign(cent), cent


def qgc(q_ctx, k, n_clusters=C_CLUSTERS):
    """QGC of one unit: (assignment [L], U32 [d, 32]) with U16 = U32[:, :16]."""
    u32 = round_to_f32(query_basis(q_ctx, R_QGS)[0])
    a, _ = kmeans(np.asarray(k, dtype=np.float64) @ u32[:, :R_QGC], n_clusters)
    return a, u32


def cluster_stats(k, v, assign, n_clusters=C_CLUSTERS):
    """Per cluster: count n [C], sums of keys and values [C, d] and of the
    squared keys (elementwise) [C, d]."""
    d = k.shape[1]
    n = np.zeros(n_clusters, dtype=np.int64)
    sk = np.zeros((n_clusters, d))
    sv = np.zeros((n_clusters, d))
    sk2 = np.zeros((n_clusters, d))
    for c in range(n_clusters):
        mem = assign == c
        n[c] = int(mem.sum())
        sk[c] = k[mem].sum(axis=0)
        sv[c] = v[mem].sum(axis=0)
        sk2[c] = (k[mem] ** 2).sum(axis=0)
    return {"n": n, "sum_k": sk, "sum_v": sv, "sum_k2": sk2}


def cluster_errors(q, cs, scale):
    """ErrorGate's estimated weight error of each cluster (module docstring)."""
    n = cs["n"].astype(np.float64)
    live = n > 0
    mean = np.zeros_like(cs["sum_k"])
    var = np.zeros_like(cs["sum_k"])
    mean[live] = cs["sum_k"][live] / n[live, None]
    var[live] = np.maximum(cs["sum_k2"][live] / n[live, None] - mean[live] ** 2, 0.0)
    mu = scale * (q @ mean.T)                                   # [G, C]
    sig2 = scale ** 2 * ((q ** 2) @ var.T)                      # [G, C]
    m = np.max(np.where(live[None, :], mu + sig2 / 2, -np.inf), axis=1, keepdims=True)
    mass = np.where(live[None, :], n[None, :] * np.exp(mu + sig2 / 2 - m), 0.0)
    err = np.where(live[None, :], n[None, :] * np.exp(mu - m) * np.expm1(sig2 / 2), 0.0)
    return (err / mass.sum(axis=1, keepdims=True)).sum(axis=0)


def errorgate(err, n, budget):
    """Integer split of `budget` tokens over the clusters (module docstring)."""
    err = np.asarray(err, dtype=np.float64)
    n = np.asarray(n, dtype=np.int64)
    C = len(n)
    top = err.max() if len(err) else 0.0
    w = np.zeros(C, dtype=np.int64) if top <= 0 else np.array([int(np.rint(x / top * 2.0 ** 30)) for x in err])
    W = int(w.sum())
    budget = int(min(budget, int(n.sum())))
    if W > 0:
        q = np.minimum(n, (budget * w) // W)
        rem = (budget * w) % W
    else:
        q = np.zeros(C, dtype=np.int64)
        rem = np.zeros(C, dtype=np.int64)
    left = budget - int(q.sum())
    order = sorted(range(C), key=lambda c: (-int(rem[c]), c))
    while left > 0:
        gave = False
        for c in order:
            if left == 0:
                break
            if q[c] < n[c]:
                q[c] += 1
                left -= 1
                gave = True
        if not gave:
            break
    return q


def qgs_codes(k, u32, exact=True):
    """int8 codes [L, 32] and fp32 scales [L] of the keys in the QGS basis
    (fp32 entries).  exact: each coordinate the exact sum of the exact
    products rounded once (math.fsum); otherwise a plain fp64 matrix product
    (for large caches, where the codes only serve as inputs)."""
    k = np.asarray(k, dtype=np.float64)
    L, r = k.shape[0], u32.shape[1]
    if exact:
        z = np.empty((L, r))
        for j in range(L):
            for i in range(r):
                z[j, i] = math.fsum(k[j] * u32[:, i])
    else:
        z = k @ u32
    amax = np.abs(z).max(axis=1)
    sig = round_to_f32(amax / 127.0)
    code = np.zeros((L, r), dtype=np.int64)
    nz = sig > 0
    code[nz] = np.clip(np.rint(z[nz] / sig[nz, None]), -127, 127).astype(np.int64)
    return code, sig


def qgs_query(q, u32):
    """The group's projected query coded to 16 bits (module docstring)."""
    qbar = np.asarray(q, dtype=np.float64).sum(axis=0)
    p = np.array([math.fsum(qbar * u32[:, i]) for i in range(u32.shape[1])])
    top = np.abs(p).max()
    if top == 0:
        return np.zeros(len(p), dtype=np.int64)
    sq = top / 32767.0
    return np.clip(np.rint(p / sq), -32767, 32767).astype(np.int64)


def qgs_scores(qq, code, sig):
    """fp32(sigma_j * (qq . code_j)) for every token."""
    dot = code @ qq                                   # exact integers
    return round_to_f32(sig * dot.astype(np.float64))


def select_tokens(scores, assign, q_per_cluster):
    """Each cluster's top q_b tokens by (score desc, index asc); returns the
    read positions in ascending order."""
    out = []
    for c, qb in enumerate(q_per_cluster):
        if qb <= 0:
            continue
        mem = np.flatnonzero(assign == c)
        order = np.lexsort((mem, -scores[mem]))
        out.extend(mem[order[:qb]].tolist())
    return np.array(sorted(out), dtype=np.int64)


def multi_proxy(q, k, v, read, assign, cs, scale):
    """Stage 04: one softmax over the exact logits of the read tokens and one
    count-aware proxy per cluster for its unread members (logit s q . Kbar' +
    ln n', value Vbar', both means over the unread members = cluster sums
    minus the read members')."""
    read = np.asarray(read, dtype=np.int64)
    logits = [scale * (q @ k[read].T)]
    values = [v[read]]
    for c in range(len(cs["n"])):
        mem_read = read[assign[read] == c] if len(read) else read
        n_un = int(cs["n"][c]) - len(mem_read)
        if n_un <= 0:
            continue
        kb = (cs["sum_k"][c] - k[mem_read].sum(axis=0)) / n_un
        vb = (cs["sum_v"][c] - v[mem_read].sum(axis=0)) / n_un
        logits.append((scale * (q @ kb) + math.log(n_un))[:, None])
        values.append(vb[None, :])
    lg = np.concatenate(logits, axis=1)
    vals = np.concatenate(values, axis=0)
    m = lg.max(axis=1, keepdims=True)
    w = np.exp(lg - m)
    return (w @ vals) / w.sum(axis=1, keepdims=True)


def step(q, k, v, assign, u32, cs, codes, sig, scale, budget):
    """One decode step of the pipeline: (read positions, per-cluster reads,
    output [G, d])."""
    err = cluster_errors(q, cs, scale)
    qb = errorgate(err, cs["n"], budget)
    scores = qgs_scores(qgs_query(q, u32), codes, sig)
    read = select_tokens(scores, assign, qb)
    return read, qb, multi_proxy(q, k, v, read, assign, cs, scale)
