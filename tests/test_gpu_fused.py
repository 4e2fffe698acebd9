"""GPU checks of the fused step kernel (selection and decode of a unit in one
CTA): it is taken exactly where its conditions hold, its outputs and
selections equal the two-kernel path bit for bit, and sampled units match
the oracle."""
import os

import numpy as np
import pytest
import torch

import synth
import kv_cache_residual_b200 as sa
from parity_util import REL_L2_OUT, OracleUnit, f64, rel_l2

pytestmark = pytest.mark.gpu

MODES = ("drop", "resa", "proxy", "sample")

# 38 x 4 = 152 units: one CTA per unit, one decode chunk per unit
WIDE = synth.scaled(synth.WORKLOADS["llama"], B=38, Hq=16, Hkv=4, L=2048, n_hh=8, seed=21)


@pytest.fixture(scope="module", autouse=True)
def fused_on():
    """The fused kernel is opt-in: on for this module only."""
    old = os.environ.get("SA_FUSED_STEP")
    os.environ["SA_FUSED_STEP"] = "1"
    yield
    if old is None:
        del os.environ["SA_FUSED_STEP"]
    else:
        os.environ["SA_FUSED_STEP"] = old


@pytest.fixture(scope="module")
def wide():
    dev = torch.device("cuda")
    data = synth.make_batch(WIDE, device=dev, steps=2)
    st = sa.prefill_stats(data["q_ctx"], data["k"], data["v"])
    torch.cuda.synchronize()
    return data, st


def _sp(k_blocks=6, sample_b=48, step=1):
    return sa.SelectParams(sink=WIDE.sink, local=WIDE.local, k_blocks=k_blocks, sample_b=sample_b,
                           sample_cap=sample_b, seed=99, step=step)


def test_fused_taken_where_it_applies(wide):
    data, _ = wide
    q, k = data["q"][0], data["k"]
    for m in MODES:
        assert sa.step_fused(q, k, _sp(), m)
    os.environ["SA_FUSED_STEP"] = "0"
    assert not sa.step_fused(q, k, _sp(), "resa")                       # opt-in only
    os.environ["SA_FUSED_STEP"] = "1"
    assert not sa.step_fused(q, k, _sp(k_blocks=40), "resa")            # k above the warp lists
    assert not sa.step_fused(q, k, _sp(sample_b=300), "sample")         # draws beyond the shared list
    small = synth.scaled(synth.WORKLOADS["llama"], B=2, Hq=16, Hkv=4, L=2048, n_hh=8, seed=22)
    ks = torch.empty(small.B, small.Hkv, small.L, small.d, dtype=torch.bfloat16, device="cuda")
    assert not sa.step_fused(q[:2], ks, _sp(), "resa")                  # too few units for a CTA each


@pytest.mark.parametrize("k_blocks", [6, 32, 40])
def test_fused_equals_two_kernels(wide, k_blocks):
    data, st = wide
    q, K, V = data["q"][1], data["k"], data["v"]
    for m in MODES:
        sp = _sp(k_blocks=k_blocks)
        sel = sa.select(q, st, sp)
        want = sa.decode(q, K, V, st, sel, sp, mode=m)
        got, sel2 = sa.step(q, K, V, st, sp, mode=m)
        torch.cuda.synchronize()
        assert torch.equal(sel.blk_idx, sel2.blk_idx) and torch.equal(sel.samp_idx, sel2.samp_idx)
        assert torch.equal(sel.samp_count, sel2.samp_count)
        assert torch.equal(got, want), (m, k_blocks)


def test_fused_against_oracle(wide):
    data, st = wide
    q = data["q"][0]
    sp = _sp()
    outs = {}
    for m in MODES:
        outs[m], sel = sa.step(q, data["k"], data["v"], st, sp, mode=m)
    torch.cuda.synchronize()
    for b, g in [(0, 0), (17, 2), (37, 3)]:
        o = OracleUnit(data, b, g, WIDE.G, WIDE.dtype)
        qq = o.q(q)
        blocks, idx, tail = o.select(qq, sp)
        np.testing.assert_array_equal(sel.blk_idx[b, g].cpu().numpy(), blocks)
        pos = o.draws(tail, sp, 48)
        np.testing.assert_array_equal(sel.samp_idx[b, g].cpu().numpy(), pos)
        for m in MODES:
            e = rel_l2(f64(outs[m][b, g * WIDE.G:(g + 1) * WIDE.G]), o.out(m, qq, idx, pos=pos))
            assert e < REL_L2_OUT, (b, g, m, e)
