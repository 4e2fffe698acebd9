"""The decode step captured once in a CUDA graph and replayed: sa_step's two
kernels (the decode a programmatic dependent of the selection) record into
the graph with their dependency, reuse the caller's workspace, and a replay
with a new query in the captured buffer gives exactly the eager result."""
import pytest
import torch

import synth
import kv_cache_residual_b200 as sa

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode", ["resa", "sample"])
def test_step_replayed_from_a_cuda_graph(mode):
    dev = torch.device("cuda")
    w = synth.scaled(synth.WORKLOADS["llama"], B=2, Hq=8, Hkv=2, L=4096, n_hh=16, seed=71)
    data = synth.make_batch(w, device=dev, steps=4)
    st = sa.prefill_stats(data["q_ctx"], data["k"], data["v"])
    sp = sa.SelectParams(sink=w.sink, local=w.local, k_blocks=16, sample_b=64, sample_cap=64, seed=5, step=2)
    q_static = data["q"][0].clone()
    out_static = torch.empty(w.B, w.Hq, w.d, dtype=torch.float32, device=dev)
    sel_static = sa.Selection(w.B, w.Hkv, sp.k_blocks, 64, dev)
    # eager warm-up: loads the kernels and allocates the workspace outside capture
    sa.step(q_static, data["k"], data["v"], st, sp, mode=mode, selection=sel_static, out=out_static)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        sa.step(q_static, data["k"], data["v"], st, sp, mode=mode, selection=sel_static, out=out_static)
    for t in range(1, 4):
        q_static.copy_(data["q"][t])
        graph.replay()
        torch.cuda.synchronize()
        out, sel = sa.step(data["q"][t], data["k"], data["v"], st, sp, mode=mode)
        torch.cuda.synchronize()
        assert torch.equal(sel.blk_idx, sel_static.blk_idx), t
        assert torch.equal(sel.samp_count, sel_static.samp_count), t
        assert torch.equal(sel.samp_idx[..., :64], sel_static.samp_idx[..., :64]) or mode != "sample", t
        assert torch.equal(out, out_static), t
