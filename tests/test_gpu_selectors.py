"""GPU parity of the two alternative block scores (max over the group's heads;
Quest's per-block key minimum and maximum): the per-block bounds bit-exact,
the chosen blocks and draws bit-exact against the oracle's selection with the
same score, outputs of every mode within the bar on those index sets.  Cases:
the tiny fp32 workload, small bf16 batches of every group size, the
one-sequence and 32-sequence 32K layers and the 128K cache at full size on
sampled units, exact ties whose band exceeds the 512 members ranked in
shared memory, near-equal scores, and the cache growing by appends."""
import zlib

import numpy as np
import pytest
import torch

import kv_cache_residual_b200 as sa
import synth
from oracle import select as osel
from oracle import stats as ostats
from parity_util import REL_L2_OUT, OracleUnit, f64, rel_l2

pytestmark = pytest.mark.gpu

SCORES = ("mean_max", "quest")


def _batch(w, steps=2):
    dev = torch.device("cuda")
    data = synth.make_batch(w, device=dev, steps=steps)
    st = sa.prefill_stats(data["q_ctx"], data["k"], data["v"], minmax=True)
    return data, st


def _check_unit(data, st, w, b, g, sp, score, sel, q_step, modes=(), outs=None):
    ou = OracleUnit(data, b, g, w.G, w.dtype)
    q = ou.q(q_step)
    blocks, idx, tail = osel.select_unit(q, ou.st["blk_mean"], w.L, sp.sink, sp.local, sp.k_blocks,
                                         score=score, st=ou.st)
    got = sel.blk_idx[b, g].cpu().numpy()
    assert got[: len(blocks)].tolist() == blocks.tolist(), (score, b, g)
    n = int(sel.samp_count[b, g])
    pos = ou.draws(tail, sp, n) if n > 0 else None
    if n > 0:
        assert sel.samp_idx[b, g, :n].cpu().tolist() == pos.tolist()
    for m in modes:
        want = ou.out(m, q, idx, pos=pos if m == "sample" else None)
        o = outs[m][b, g * w.G:(g + 1) * w.G]
        assert rel_l2(f64(o), want) <= REL_L2_OUT, (score, m, b, g)


def test_block_minmax_bit_exact():
    w = synth.scaled(synth.WORKLOADS["llama"], B=2, L=4096)
    data, st = _batch(w, 1)
    for b in range(w.B):
        for g in range(w.Hkv):
            mn, mx = ostats.block_minmax(f64(data["k"][b, g]))
            assert np.array_equal(f64(st.blk_min[b, g]), mn)
            assert np.array_equal(f64(st.blk_max[b, g]), mx)
    wt = synth.WORKLOADS["tiny"]
    dt, stt = _batch(wt, 1)
    mn, mx = ostats.block_minmax(f64(dt["k"][0, 0]))
    assert np.array_equal(f64(stt.blk_min[0, 0]), mn) and np.array_equal(f64(stt.blk_max[0, 0]), mx)


@pytest.mark.parametrize("score", SCORES)
def test_tiny_every_mode(score):
    w = synth.WORKLOADS["tiny"]
    data, st = _batch(w, 3)
    for step in range(3):
        sp = sa.SelectParams(sink=w.sink, local=w.local, k_blocks=w.k_blocks, sample_b=w.sample_b,
                             sample_cap=w.sample_b, seed=11, step=step, score=score)
        q = data["q"][step]
        sel = sa.select(q, st, sp)
        outs = {m: sa.decode(q, data["k"], data["v"], st, sel, sp, mode=m) for m in sa.MODES}
        torch.cuda.synchronize()
        _check_unit(data, st, w, 0, 0, sp, score, sel, q, modes=tuple(sa.MODES), outs=outs)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("score", SCORES)
def test_small_bf16_batches_through_step(score, G):
    base = synth.WORKLOADS["llama"]
    Hkv = 2
    w = synth.scaled(base, B=3, Hq=G * Hkv, Hkv=Hkv, L=4096, n_hh=16, seed=500 + G)
    data, st = _batch(w, 2)
    for step in range(2):
        for k_blocks in (8, 40):
            sp = sa.SelectParams(sink=w.sink, local=w.local, k_blocks=k_blocks, sample_b=32, sample_cap=32,
                                 seed=5, step=step, score=score)
            q = data["q"][step]
            outs = {}
            for m in ("resa", "proxy", "sample"):
                outs[m], sel = sa.step(q, data["k"], data["v"], st, sp, mode=m)
            torch.cuda.synchronize()
            for b in range(w.B):
                for g in range(w.Hkv):
                    _check_unit(data, st, w, b, g, sp, score, sel, q, modes=("resa", "proxy", "sample"),
                                outs=outs)


@pytest.mark.parametrize("score", SCORES)
def test_llama_layer_full_size(score):
    w = synth.WORKLOADS["llama"]
    data, st = _batch(w, 1)
    q = data["q"][0]
    for read in w.read_fracs:
        sp = sa.SelectParams(sink=w.sink, local=w.local, k_blocks=w.k_blocks_for(read), seed=3, step=0, score=score)
        out, sel = sa.step(q, data["k"], data["v"], st, sp, mode="resa")
        torch.cuda.synchronize()
        for g in (0, 3, 7):
            _check_unit(data, st, w, 0, g, sp, score, sel, q, modes=("resa",), outs={"resa": out})


@pytest.mark.parametrize("score", SCORES)
def test_batched_full_size_sampled_units(score):
    w = synth.WORKLOADS["batched"]
    data, st = _batch(w, 1)
    q = data["q"][0]
    sp = sa.SelectParams(sink=w.sink, local=w.local, k_blocks=w.k_blocks_for(0.01), seed=3, step=0, score=score)
    out, sel = sa.step(q, data["k"], data["v"], st, sp, mode="resa")
    torch.cuda.synchronize()
    for b, g in ((0, 0), (17, 5), (31, 7)):
        _check_unit(data, st, w, b, g, sp, score, sel, q, modes=("resa",), outs={"resa": out})


def test_long_context_full_size_sampled_units():
    w = synth.scaled(synth.WORKLOADS["long"], B=2)
    data, st = _batch(w, 1)
    q = data["q"][0]
    for score in SCORES:
        for read in w.read_fracs:
            sp = sa.SelectParams(sink=w.sink, local=w.local, k_blocks=w.k_blocks_for(read), seed=9, step=0,
                                 score=score)
            sel = sa.select(q, st, sp)
            torch.cuda.synchronize()
            for b, g in ((0, 1), (1, 6)):
                _check_unit(data, st, w, b, g, sp, score, sel, q)


@pytest.mark.parametrize("pattern", ["ties", "near"])
@pytest.mark.parametrize("score", SCORES)
def test_ties_and_wide_bands(score, pattern):
    """Summaries written by hand: rows drawn from three vectors (exact ties,
    lowest indices win; the band of the tied group exceeds the 512 members
    ranked in shared memory) or one row plus a 1e-3 perturbation (near-equal
    scores, rescored exactly)."""
    B, Hq, Hkv, d, L = 2, 8, 2, 128, 32768
    G = Hq // Hkv
    dev = torch.device("cuda")
    gen = torch.Generator().manual_seed(zlib.crc32(("%s/%s" % (score, pattern)).encode()))
    nb = L // 16
    if pattern == "ties":
        base = torch.randn(B, Hkv, 3, d, generator=gen)
        pick = torch.randint(0, 3, (B, Hkv, nb), generator=gen)
        rows = torch.gather(base, 2, pick.unsqueeze(-1).expand(B, Hkv, nb, d))
    else:
        rows = torch.randn(B, Hkv, 1, d, generator=gen) + 1e-3 * torch.randn(B, Hkv, nb, d, generator=gen)
    rows = rows.to(torch.bfloat16)
    st = sa.Stats(B, Hq, Hkv, L, d, torch.bfloat16, dev, minmax=True)
    st.blk_mean.copy_(rows.to(dev))
    # quest bounds: min = the row, max = the row + a block-dependent spread
    st.blk_min.copy_(rows.to(dev))
    spread = (0.5 * torch.rand(B, Hkv, nb, 1, generator=gen)).to(torch.bfloat16).float()
    st.blk_max.copy_((rows.float() + (spread if pattern == "near" else 0.25)).to(torch.bfloat16).to(dev))
    q = torch.randn(B, Hq, d, generator=gen).to(torch.bfloat16)
    cand = osel.candidate_blocks(L, 64, 128)
    for k_blocks in (8, 32, 100):
        sp = sa.SelectParams(sink=64, local=128, k_blocks=k_blocks, score=score)
        sel = sa.select(q.to(dev), st, sp)
        torch.cuda.synchronize()
        for b in range(B):
            for g in range(Hkv):
                qq = f64(q[b, g * G:(g + 1) * G])
                ost = {"blk_mean": f64(st.blk_mean[b, g]), "blk_min": f64(st.blk_min[b, g]),
                       "blk_max": f64(st.blk_max[b, g])}
                want = osel.top_blocks(osel.scores_for(score, qq, ost, cand), cand, k_blocks)
                assert sel.blk_idx[b, g, :k_blocks].cpu().tolist() == want.tolist(), (score, pattern, k_blocks)
        if pattern == "ties":
            # a third of the candidates tie with the k-th: the band is wider than
            # the 512 members ranked in shared memory (exact keys in the workspace)
            assert int(sel.n_rescored.max()) > 512


def test_append_keeps_block_bounds():
    w = synth.scaled(synth.WORKLOADS["llama"], B=1, Hq=8, Hkv=2, L=2048 + 32)
    dev = torch.device("cuda")
    data = synth.make_batch(w, device=dev, steps=1)
    L0 = 2048
    k, v = data["k"], data["v"]
    kc, vc = torch.zeros_like(k), torch.zeros_like(v)
    kc[:, :, :L0] = k[:, :, :L0]
    vc[:, :, :L0] = v[:, :, :L0]
    st = sa.prefill_stats(data["q_ctx"][:, :, :L0].contiguous(), kc, vc, minmax=True)
    length = L0
    for t in range(L0, L0 + 32):
        length = sa.append(k[:, :, t].contiguous(), v[:, :, t].contiguous(), kc, vc, st, length)
    torch.cuda.synchronize()
    for g in range(w.Hkv):
        mn, mx = ostats.block_minmax(f64(k[0, g, :length]))
        assert np.array_equal(f64(st.blk_min[0, g, : length // 16]), mn)
        assert np.array_equal(f64(st.blk_max[0, g, : length // 16]), mx)
