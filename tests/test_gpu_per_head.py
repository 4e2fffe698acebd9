"""GPU parity of per-query-head sampling (vAttention samples and sets the
budget per head): every query head draws from its own stream, gets its own
budget from its own base sample, and its draws are weighted n_T / b_h in its
softmax alone, while the exactly read set stays the KV head's.  Draws are
compared bit for bit, budgets as integers (a difference allowed only where
the real-valued budget lies within 1e-9 of an integer), outputs within the
bar."""
import math

import numpy as np
import pytest
import torch

import synth
import kv_cache_residual_b200 as sa
from oracle import budget as obudget
from oracle import modes as omodes
from oracle import rng as orng
from parity_util import REL_L2_OUT, OracleUnit, f64, rel_l2

pytestmark = pytest.mark.gpu

RULES = {"clt": obudget.clt_budget, "clt_search": obudget.clt_budget_search, "hoeffding": obudget.hoeffding_budget}


def _check(w, data, q, sel, out, sp, units, rule=None):
    counts = sel.samp_count.cpu().numpy()
    eps, delta = float(np.float32(sp.eps)), float(np.float32(sp.delta))
    for b, g in units:
        o = OracleUnit(data, b, g, w.G, w.dtype)
        qq = o.q(q)
        blocks, idx, tail = o.select(qq, sp)
        np.testing.assert_array_equal(sel.blk_idx[b, g].cpu().numpy()[:len(blocks)], blocks)
        pos = []
        for h in range(w.G):
            hq = g * w.G + h
            n = int(counts[b, hq])
            if rule is not None:
                base = orng.sample_positions(sp.seed, b, hq, sp.step, tail, sp.clt_base)
                want, det = RULES[rule](qq[h:h + 1], o.k, o.v, idx, base, o.scale, eps, delta, len(tail))
                want = min(want, sp.sample_cap)
                if n != want:
                    best = det["b_real"] if rule == "clt_search" else max(max(det["b_N"]), max(det["b_D"]))
                    assert math.isfinite(best) and abs(best - round(best)) <= 1e-9 * best, (b, hq, n, want)
            else:
                assert n == min(sp.sample_b, len(tail))
            p = orng.sample_positions(sp.seed, b, hq, sp.step, tail, n)
            np.testing.assert_array_equal(sel.samp_idx[b, hq].cpu().numpy()[:n], p)
            pos.append(p)
        want = omodes.sample_per_head(qq, o.k, o.v, idx, pos, o.scale)
        e = rel_l2(f64(out[b, g * w.G:(g + 1) * w.G]), want)
        assert e < REL_L2_OUT, (b, g, e)
    return counts


def test_tiny_fixed_draws_per_head():
    w = synth.WORKLOADS["tiny"]
    dev = torch.device("cuda")
    data = synth.make_batch(w, device=dev, steps=2)
    st = sa.prefill_stats(data["q_ctx"], data["k"], data["v"])
    for step in range(2):
        sp = sa.SelectParams(sink=w.sink, local=w.local, k_blocks=w.k_blocks, sample_b=48, sample_cap=64, seed=8,
                             step=step, per_head=True)
        q = data["q"][step]
        sel = sa.select(q, st, sp)
        out = sa.decode(q, data["k"], data["v"], st, sel, sp, mode="sample")
        torch.cuda.synchronize()
        _check(w, data, q, sel, out, sp, [(0, 0)])


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_bf16_fixed_draws_per_head(G):
    Hkv = 2
    w = synth.scaled(synth.WORKLOADS["llama"], B=2, Hq=G * Hkv, Hkv=Hkv, L=4096, n_hh=16, seed=700 + G)
    dev = torch.device("cuda")
    data = synth.make_batch(w, device=dev, steps=1)
    st = sa.prefill_stats(data["q_ctx"], data["k"], data["v"])
    q = data["q"][0]
    for b_draw, cap in ((40, 64), (100, 100)):
        sp = sa.SelectParams(sink=w.sink, local=w.local, k_blocks=8, sample_b=b_draw, sample_cap=cap, seed=21,
                             step=0, per_head=True)
        out, sel = sa.step(q, data["k"], data["v"], st, sp, mode="sample")
        torch.cuda.synchronize()
        _check(w, data, q, sel, out, sp, [(b, g) for b in range(w.B) for g in range(w.Hkv)])


@pytest.mark.parametrize("rule", list(RULES))
def test_budget_per_head(rule):
    w = synth.scaled(synth.WORKLOADS["flat"], B=2, Hq=8, Hkv=2, L=8192, seed=43)
    dev = torch.device("cuda")
    data = synth.make_batch(w, device=dev, steps=1)
    st = sa.prefill_stats(data["q_ctx"], data["k"], data["v"])
    q = data["q"][0]
    eps = 0.8
    sp = sa.SelectParams(sink=w.sink, local=w.local, k_blocks=w.k_blocks_for(0.02), sample_cap=8192, clt_base=64,
                         eps=eps, delta=0.1, seed=5, step=0, budget=rule, per_head=True)
    out, sel = sa.step(q, data["k"], data["v"], st, sp, mode="sample")
    torch.cuda.synchronize()
    counts = _check(w, data, q, sel, out, sp, [(b, g) for b in range(w.B) for g in range(w.Hkv)], rule=rule)
    assert (counts >= 64).all()
    if rule != "hoeffding":                               # (the conservative bound asks for the whole tail here)
        assert len(np.unique(counts)) > 1                 # the heads' budgets differ


def test_other_modes_ignore_per_head_draws():
    w = synth.scaled(synth.WORKLOADS["llama"], B=2, Hq=8, Hkv=2, L=4096, n_hh=16, seed=77)
    dev = torch.device("cuda")
    data = synth.make_batch(w, device=dev, steps=1)
    st = sa.prefill_stats(data["q_ctx"], data["k"], data["v"])
    q = data["q"][0]
    for m in ("drop", "resa", "proxy"):
        a, _ = sa.step(q, data["k"], data["v"], st, sa.SelectParams(k_blocks=8, sample_b=32, sample_cap=32), mode=m)
        bb, _ = sa.step(q, data["k"], data["v"], st,
                        sa.SelectParams(k_blocks=8, sample_b=32, sample_cap=32, per_head=True), mode=m)
        torch.cuda.synchronize()
        assert torch.equal(a, bb), m
