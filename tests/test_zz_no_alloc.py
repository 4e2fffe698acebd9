"""sa_select_noalloc: the selection entry point for callers that cannot
allocate device memory (it keeps its scratch in a fixed array inside the
library).  Its results must be those of sa_select with a caller workspace,
call after call.  This file is collected last so that a run stopping at the
first failure has already run every other test; it also passes on its own in
a fresh process."""
import ctypes

import pytest
import torch

import synth
import kv_cache_residual_b200 as sa

pytestmark = pytest.mark.gpu


def _noalloc_select(q, stats, params, scale=0.0, k=None, v=None):
    B, Hq, d = q.shape
    Hkv, L = stats.blk_mean.shape[1], stats.blk_mean.shape[2] * 16
    shape = sa.sa_shape(B, Hq, Hkv, d, L, sa._dtype_code(q))
    cp = params.c()
    sel = sa.Selection(B, Hkv, params.k_blocks, cp.sample_cap, q.device)
    st = stats.c()
    c_sel = sel.c()
    status = sa._lib().sa_select_noalloc(ctypes.byref(shape), ctypes.byref(cp), sa._ptr(q), ctypes.byref(st),
                                         sa._ptr(k), sa._ptr(v), ctypes.byref(c_sel), float(scale), sa._stream())
    assert status == sa.SA_OK, sa._lib().sa_status_string(status)
    return sel


@pytest.mark.parametrize("wname,B", [("tiny", 1), ("llama", 2), ("batched", 20)])
def test_noalloc_select_matches_workspace_select_twice(wname, B):
    """Two calls in a row (different steps) against sa_select: chosen blocks,
    draws and draw counts identical (index results, compared exactly)."""
    assert torch.cuda.is_available()
    w = synth.scaled(synth.WORKLOADS[wname], B=B, L=min(synth.WORKLOADS[wname].L, 8192))
    dev = torch.device("cuda")
    data = synth.make_batch(w, device=dev, steps=2)
    st = sa.prefill_stats(data["q_ctx"], data["k"], data["v"])
    kb = w.k_blocks if w.k_blocks is not None else 8
    for step in range(2):
        sp = sa.SelectParams(sink=w.sink, local=w.local, k_blocks=kb, sample_b=64, sample_cap=64,
                             seed=99, step=step)
        q = data["q"][step]
        want = sa.select(q, st, sp)
        got = _noalloc_select(q, st, sp)
        torch.cuda.synchronize()
        assert torch.equal(got.blk_idx, want.blk_idx)
        assert torch.equal(got.samp_count, want.samp_count)
        assert torch.equal(got.samp_idx, want.samp_idx)


def test_noalloc_clt_budget_matches_workspace_select_twice():
    """The sampling budget path through the fixed array (its completion
    tickets and per-split fp64 records): flat keys, base sample of 64 draws,
    two calls in a row against sa_select."""
    w = synth.scaled(synth.WORKLOADS["flat"], B=2, L=8192)
    dev = torch.device("cuda")
    data = synth.make_batch(w, device=dev, steps=2)
    st = sa.prefill_stats(data["q_ctx"], data["k"], data["v"])
    for step in range(2):
        sp = sa.SelectParams(sink=w.sink, local=w.local, k_blocks=w.k_blocks_for(0.05), sample_cap=2048,
                             clt_base=64, eps=0.1, delta=0.05, seed=7, step=step)
        q = data["q"][step]
        want = sa.select(q, st, sp, k=data["k"], v=data["v"])
        got = _noalloc_select(q, st, sp, k=data["k"], v=data["v"])
        torch.cuda.synchronize()
        assert torch.equal(got.blk_idx, want.blk_idx)
        assert torch.equal(got.samp_count, want.samp_count)
        assert int(want.samp_count.min()) > 64            # the budget asked for more than the base sample
        for u in range(w.B * w.Hkv):
            b, g = divmod(u, w.Hkv)
            n = int(want.samp_count[b, g])
            assert torch.equal(got.samp_idx[b, g, :n], want.samp_idx[b, g, :n])


def test_noalloc_rejected_call_enqueues_nothing():
    """A call whose arguments are wrong (a misaligned query) returns before
    touching the fixed array or the stream."""
    B, Hq, Hkv, d, L = 1, 4, 1, 64, 2048
    shape = sa.sa_shape(B, Hq, Hkv, d, L, sa.SA_BF16)
    cp = sa.SelectParams(k_blocks=4).c()
    st = sa.sa_stats(*([0x10000] * 10))
    sel = sa.sa_selection(0x10000, 0x10000, 0x10000, 0)
    status = sa._lib().sa_select_noalloc(ctypes.byref(shape), ctypes.byref(cp), ctypes.c_void_p(0x10002),
                                         ctypes.byref(st), None, None, ctypes.byref(sel), 0.0, None)
    assert status == sa.SA_ERR_INVALID_ARG


def test_noalloc_rejects_shapes_beyond_its_array():
    B, Hq, Hkv, d, L = 64, 32, 8, 128, 131072      # selection workspace far above 8 MiB
    shape = sa.sa_shape(B, Hq, Hkv, d, L, sa.SA_BF16)
    cp = sa.SelectParams(k_blocks=8).c()
    assert sa._lib().sa_workspace_size(ctypes.byref(shape), ctypes.byref(cp), sa.OP_SELECT) > (8 << 20)
    p = ctypes.c_void_p(0x10000)
    st = sa.sa_stats(*([0x10000] * 10))
    sel = sa.sa_selection(0x10000, 0x10000, 0x10000, 0)
    status = sa._lib().sa_select_noalloc(ctypes.byref(shape), ctypes.byref(cp), p, ctypes.byref(st), None, None,
                                         ctypes.byref(sel), 0.0, None)
    assert status == sa.SA_ERR_WORKSPACE
