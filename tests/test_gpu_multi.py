"""GPU parity of the OpenAttention multi-proxy path: the QGS codes and the
cluster sums from a basis and an assignment, and each decode step (ErrorGate
split, per-cluster QGS top-q, one proxy per cluster) against the oracle run
on the same inputs.  The clusters come from the oracle's QGC (query basis
and k-means) and are handed to the kernels, so that the per-step path is
compared on identical clusters; budgets per cluster and read sets are
compared exactly, outputs within the bar."""
import math

import numpy as np
import pytest
import torch

import kv_cache_residual_b200 as sa
import synth
from oracle import openattn as OA
from oracle.numerics import round_to_f32
from parity_util import REL_L2_OUT, f64, rel_l2

pytestmark = pytest.mark.gpu


def _oracle_clusters(data, b, g, G, C, exact_codes):
    k = f64(data["k"][b, g])
    qctx = f64(data["q_ctx"][b, g * G:(g + 1) * G])
    a, u32 = OA.qgc(qctx, k, C)
    code, sig = OA.qgs_codes(k, u32, exact=exact_codes)
    cs = OA.cluster_stats(k, f64(data["v"][b, g]), a, C)
    return a, u32, code, sig, cs


def _order(a, C):
    """The cluster-major order of the positions (ascending within a cluster)
    and the clusters' starts."""
    order = np.argsort(a, kind="stable")
    start = np.concatenate([[0], np.cumsum(np.bincount(a, minlength=C))])
    return order, start


def _to_gpu(cl, b, g, a, u32, code, sig, cs):
    dev = cl.basis.device
    order, start = _order(a, cl.n_clusters)
    cl.basis[b, g] = torch.from_numpy(u32.T.copy()).float().to(dev)
    cl.assign[b, g, :len(a)] = torch.from_numpy(a.astype(np.uint8)).to(dev)
    cl.order[b, g, :len(a)] = torch.from_numpy(order.astype(np.int32)).to(dev)
    cl.start[b, g] = torch.from_numpy(start.astype(np.int32)).to(dev)
    cl.codes[b, g, :len(a)] = torch.from_numpy(code[order].astype(np.int8)).to(dev)
    cl.scales[b, g, :len(a)] = torch.from_numpy(sig[order]).float().to(dev)
    cl.count[b, g] = torch.from_numpy(cs["n"].astype(np.int32)).to(dev)
    for f in ("sum_k", "sum_v", "sum_k2"):
        getattr(cl, f)[b, g] = torch.from_numpy(cs[f]).float().to(dev)


def _cs32(cs):
    return {"n": cs["n"], "sum_k": round_to_f32(cs["sum_k"]), "sum_v": round_to_f32(cs["sum_v"]),
            "sum_k2": round_to_f32(cs["sum_k2"])}


def _setup(w, C, units=None, exact_codes=False):
    dev = torch.device("cuda")
    data = synth.make_batch(w, device=dev, steps=2)
    cl = sa.Clusters(w.B, w.Hkv, w.L, w.d, C, dev)
    orc = {}
    for b in range(w.B):
        for g in range(w.Hkv):
            if units is not None and (b, g) not in units:
                continue
            orc[(b, g)] = _oracle_clusters(data, b, g, w.G, C, exact_codes)
            _to_gpu(cl, b, g, *orc[(b, g)])
    return data, cl, orc


def _check_step(w, data, cl, orc, budget, step=0):
    q = data["q"][step]
    out, read, qcnt = sa.multi_step(q, data["k"], data["v"], cl, budget)
    torch.cuda.synchronize()
    s = float(np.float32(1.0 / math.sqrt(w.d)))
    for (b, g), (a, u32, code, sig, cs) in orc.items():
        qq = f64(q[b, g * w.G:(g + 1) * w.G])
        k, v = f64(data["k"][b, g]), f64(data["v"][b, g])
        cs32 = _cs32(cs)
        rd, qb, want = OA.step(qq, k, v, a, u32, cs32, code, sig, s, budget)
        assert qcnt[b, g].cpu().tolist() == qb.tolist(), (b, g)
        got = read[b, g].cpu().numpy()
        assert (got[len(rd):] == -1).all()
        assert sorted(got[:len(rd)].tolist()) == rd.tolist(), (b, g)
        # grouped by cluster, ascending positions within each cluster
        assert list(got[:len(rd)]) == sorted(got[:len(rd)].tolist(), key=lambda j: (a[j], j))
        e = rel_l2(f64(out[b, g * w.G:(g + 1) * w.G]), want)
        assert e < REL_L2_OUT, (b, g, e)


def test_prep_codes_bit_exact_and_sums():
    w = synth.scaled(synth.WORKLOADS["llama"], B=1, Hq=8, Hkv=2, L=2048, n_hh=8, seed=900)
    data, cl, orc = _setup(w, 16, exact_codes=True)
    got = sa.Clusters(w.B, w.Hkv, w.L, w.d, 16, cl.basis.device)
    got.basis.copy_(cl.basis)
    got.assign.copy_(cl.assign)
    sa.cluster_prep(data["k"], data["v"], got, w.Hq)
    torch.cuda.synchronize()
    for (b, g), (a, u32, code, sig, cs) in orc.items():
        order, start = _order(a, 16)
        assert np.array_equal(got.order[b, g].cpu().numpy(), order)
        assert np.array_equal(got.start[b, g].cpu().numpy(), start)
        assert np.array_equal(got.codes[b, g].cpu().numpy().astype(np.int64), code[order])
        assert np.array_equal(got.scales[b, g].cpu().numpy().astype(np.float64), sig[order])
        assert got.count[b, g].cpu().tolist() == cs["n"].tolist()
        for f in ("sum_k", "sum_v", "sum_k2"):
            np.testing.assert_allclose(f64(getattr(got, f)[b, g]), cs[f], rtol=1e-6, atol=1e-4)
    # the tiny fp32 workload, d = 64
    wt = synth.WORKLOADS["tiny"]
    dt, clt, orct = _setup(wt, 8, exact_codes=True)
    gt = sa.Clusters(1, 1, wt.L, wt.d, 8, clt.basis.device)
    gt.basis.copy_(clt.basis)
    gt.assign.copy_(clt.assign)
    sa.cluster_prep(dt["k"], dt["v"], gt, wt.Hq)
    torch.cuda.synchronize()
    a, u32, code, sig, cs = orct[(0, 0)]
    order, _ = _order(a, 8)
    assert np.array_equal(gt.order[0, 0].cpu().numpy(), order)
    assert np.array_equal(gt.codes[0, 0].cpu().numpy().astype(np.int64), code[order])
    assert gt.count[0, 0].cpu().tolist() == cs["n"].tolist()


def test_tiny_steps():
    w = synth.WORKLOADS["tiny"]
    data, cl, orc = _setup(w, 16)
    for step in range(2):
        for budget in (20, 128, 2048):
            _check_step(w, data, cl, orc, budget, step)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_small_bf16_every_group_size(G):
    Hkv = 2
    w = synth.scaled(synth.WORKLOADS["llama"], B=2, Hq=G * Hkv, Hkv=Hkv, L=4096, n_hh=16, seed=910 + G)
    data, cl, orc = _setup(w, 64)
    for budget in (41, 122, 400):
        _check_step(w, data, cl, orc, budget)


def test_llama_layer_full_size_sampled_units():
    w = synth.WORKLOADS["llama"]
    data, cl, orc = _setup(w, 64, units={(0, 0), (0, 5)})
    for read in w.read_fracs:
        _check_step(w, data, cl, {u: orc[u] for u in orc}, int(read * w.L))
