"""GPU parity of cache append during decode: tokens appended one at a time
after prefill end (sa_append), with selection and decode at lengths that are
not whole blocks, against the oracle's statistics of the grown cache
(oracle.stats.grown_stats: O_Est, log_z0 and the totals over every cached
token, mu_Q and mu_K kept from prefill end).

Inputs: one synthetic sequence per batch entry, generated at the final
length; its first L0 tokens are the prefill, the rest are appended in order.
The cache tensors have room for all of them (capacity ld >= L0 + n)."""
import math

import numpy as np
import pytest
import torch

import synth
import kv_cache_residual_b200 as sa
from oracle import modes as omodes
from oracle import rng as orng
from oracle import select as osel
from oracle import stats as ostats
from parity_util import REL_L2_OUT, f64, rel_l2

pytestmark = pytest.mark.gpu

MODES = ("drop", "resa", "proxy", "sample")


def _grown_oracle(data, b, g, G, L0, L, dtype):
    """(k [L, d], v [L, d], grown statistics) of unit (b, g) at length L."""
    k = f64(data["k"][b, g, :L])
    v = f64(data["v"][b, g, :L])
    s = 1.0 / math.sqrt(k.shape[1])
    st0 = ostats.prefill_stats(f64(data["q_ctx"][b, g * G:(g + 1) * G, :L0]), k[:L0], v[:L0], s, dtype)
    return k, v, s, ostats.grown_stats(st0, k, v, s, dtype)


def _run(w, L0, n, checks, dev):
    data = synth.make_batch(w, device=dev, steps=n + 1)
    B, Hkv, Lg, d = data["k"].shape
    assert Lg == L0 + n
    ld = -(-Lg // 16) * 16
    K = torch.zeros(B, Hkv, ld, d, dtype=data["k"].dtype, device=dev)
    V = torch.zeros_like(K)
    K[:, :, :L0] = data["k"][:, :, :L0]
    V[:, :, :L0] = data["v"][:, :, :L0]
    st = sa.prefill_stats(data["q_ctx"][:, :, :L0].contiguous(), K, V)
    L = L0
    for i in range(1, n + 1):
        L = sa.append(data["k"][:, :, L].contiguous(), data["v"][:, :, L].contiguous(), K, V, st, L)
        assert L == L0 + i
        if i not in checks:
            continue
        torch.cuda.synchronize()
        assert torch.equal(K[:, :, :L], data["k"][:, :, :L]) and torch.equal(V[:, :, :L], data["v"][:, :, :L])
        # the sketch rows of the appended blocks are the ones a rebuild writes
        nb = L // 16
        code, meta = st.blk_code.clone(), st.blk_meta.clone()
        sa.block_sketch(st, w.Hq, 0, nb)
        torch.cuda.synchronize()
        assert torch.equal(code[:, :, :nb], st.blk_code[:, :, :nb]) and torch.equal(meta[:, :, :nb],
                                                                                    st.blk_meta[:, :, :nb])
        q = data["q"][i]
        sp = sa.SelectParams(sink=w.sink, local=w.local, k_blocks=8, sample_b=64,
                             sample_cap=64, seed=77, step=i)
        outs = {}
        for m in MODES:
            outs[m], sel = sa.step(q, K, V, st, sp, mode=m, length=L)
        outs["dense"] = sa.dense_decode(q, K, V, length=L)
        torch.cuda.synchronize()
        for b in range(B):
            for g in range(Hkv):
                k, v, s, gst = _grown_oracle(data, b, g, w.G, L0, L, w.dtype)
                hs = slice(g * w.G, (g + 1) * w.G)
                # refreshed statistics
                assert rel_l2(f64(st.o_est[b, hs]), gst["o_est"]) < 1e-4, (i, b, g)
                np.testing.assert_allclose(f64(st.log_z0[b, hs]), gst["log_z0"], rtol=0,
                                           atol=2e-5 * max(1.0, np.abs(gst["log_z0"]).max()))
                assert rel_l2(f64(st.sum_k[b, g]), gst["sum_k"]) < 1e-6
                assert rel_l2(f64(st.sum_v[b, g]), gst["sum_v"]) < 1e-4
                np.testing.assert_array_equal(f64(st.blk_mean[b, g, :nb]), gst["blk_mean"])
                # selection on the grown cache, bit-exact
                qq = f64(q[b, hs])
                blocks, idx, tail = osel.select_unit(qq, gst["blk_mean"], L, sp.sink, sp.local, sp.k_blocks)
                np.testing.assert_array_equal(sel.blk_idx[b, g].cpu().numpy()[:len(blocks)], blocks)
                nd = int(sel.samp_count[b, g])
                assert nd == (64 if len(tail) else 0)
                pos = orng.sample_positions(sp.seed, b, g, sp.step, tail, nd)
                np.testing.assert_array_equal(sel.samp_idx[b, g, :nd].cpu().numpy(), pos)
                for m in MODES + ("dense",):
                    want = omodes.run_mode(m, qq, k, v, idx, gst, s, pos=pos)
                    e = rel_l2(f64(outs[m][b, hs]), want)
                    assert e < REL_L2_OUT, (i, L, b, g, m, e)
    return L


def test_append_decode_loop_bf16():
    """2048 prefill tokens, 40 appended (two blocks completed on the way);
    checked after 1, 15, 16, 17, 33 and 40 appends."""
    w = synth.scaled(synth.WORKLOADS["batched"], B=2, Hq=8, Hkv=2, L=2048 + 40, seed=61)
    L = _run(w, 2048, 40, {1, 15, 16, 17, 33, 40}, torch.device("cuda"))
    assert L == 2088


def test_append_decode_loop_f32():
    """The fp32 cache path (CUDA-core kernels), tiny shape, G = 4, d = 64."""
    w = synth.scaled(synth.WORKLOADS["tiny"], L=1024 + 20, seed=62)
    L = _run(w, 1024, 20, {1, 16, 20}, torch.device("cuda"))
    assert L == 1044


def test_append_rejects_a_full_cache():
    w = synth.scaled(synth.WORKLOADS["batched"], B=1, Hq=8, Hkv=2, L=1024, seed=63)
    data = synth.make_batch(w, device=torch.device("cuda"), steps=1)
    st = sa.prefill_stats(data["q_ctx"], data["k"], data["v"])
    with pytest.raises(sa.SAError):
        sa.append(data["k"][:, :, 0].contiguous(), data["v"][:, :, 0].contiguous(), data["k"], data["v"], st, 1024)
