"""GPU parity of the selection: chosen blocks and tail draws bit-exact
against the oracle.  With enough units each gets its own CTA (the bounds stay
on chip): every dtype / d / G, k on both sides of the group top-k's limit
(32), exact ties, and score orders that stress the candidate bound.  With few
units each is split over scanning CTAs and finished by a second kernel: 64K
and 128K-token caches, k from 8 to n_cand - 1 (group top-k up to 1024 blocks,
radix select beyond), ties and near-equal scores whose band exceeds the 512
members ranked in shared memory."""
import zlib

import numpy as np
import pytest
import torch

import kv_cache_residual_b200 as sa
from oracle import rng as orng
from oracle import select as osel
from parity_util import f64

pytestmark = pytest.mark.gpu

# (dtype, d, Hq, Hkv, B, L): B * Hkv >= 148 units in every case
SHAPES = {
    "bf16_d128_g4": ("bf16", 128, 32, 8, 20, 4096),
    "bf16_d64_g8": ("bf16", 64, 16, 2, 80, 2048),
    "f32_d128_g1": ("f32", 128, 4, 4, 40, 2048),
    "f32_d64_g2": ("f32", 64, 8, 4, 38, 3104),
}
SINK, LOCAL = 64, 128


def _summaries(pattern, B, Hkv, nb, d, dt, q, G, gen):
    """Block summaries [B, Hkv, nb, d] of the given score structure."""
    if pattern == "random":
        m = torch.randn(B, Hkv, nb, d, generator=gen)
    elif pattern == "ascending":
        # score grows with the block index: a warp's list changes at every row
        qbar = q.view(B, Hkv, G, d).sum(2)
        dirn = qbar / qbar.norm(dim=-1, keepdim=True) ** 2
        ramp = torch.linspace(-4.0, 4.0, nb).view(1, 1, nb, 1)
        m = ramp * dirn.unsqueeze(2) * 16.0 + 0.01 * torch.randn(B, Hkv, nb, d, generator=gen)
    elif pattern == "near":
        # one common row plus a 1e-3 perturbation: every score lies within
        # the sketch's error bound of the others, so the band is most of the
        # candidates and the exact rescoring decides
        base = torch.randn(B, Hkv, 1, d, generator=gen)
        m = base + 1e-3 * torch.randn(B, Hkv, nb, d, generator=gen)
    elif pattern == "ties":
        # rows drawn from five distinct vectors: many exactly equal scores
        base = torch.randn(B, Hkv, 5, d, generator=gen)
        pick = torch.randint(0, 5, (B, Hkv, nb), generator=gen)
        m = torch.gather(base, 2, pick.unsqueeze(-1).expand(B, Hkv, nb, d))
    else:
        raise ValueError(pattern)
    return m.to(dt)


@pytest.mark.parametrize("pattern", ["random", "ascending", "ties", "near"])
@pytest.mark.parametrize("name", list(SHAPES))
def test_select_one_cta_per_unit(name, pattern):
    dtype, d, Hq, Hkv, B, L = SHAPES[name]
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    G = Hq // Hkv
    dev = torch.device("cuda")
    gen = torch.Generator().manual_seed(zlib.crc32(("%s/%s" % (name, pattern)).encode()))
    q = torch.randn(B, Hq, d, generator=gen).to(dt)
    nb = L // 16
    bm = _summaries(pattern, B, Hkv, nb, d, dt, q.float(), G, gen)
    st = sa.Stats(B, Hq, Hkv, L, d, dt, dev)
    st.blk_mean.copy_(bm.to(dev))
    st.kbar_absmax.copy_(bm.float().abs().amax(dim=(2, 3)).to(dev))
    st.mu_k.copy_(bm.float().mean(2).to(dev))          # the sketch's centre
    sa.block_sketch(st, Hq)
    qd = q.to(dev)
    n_cand = len(osel.candidate_blocks(L, SINK, LOCAL))
    for k in (1, 8, 32, 33, n_cand - 1):
        sp = sa.SelectParams(sink=SINK, local=LOCAL, k_blocks=k, sample_b=48, sample_cap=48, seed=77, step=3)
        sel = sa.select(qd, st, sp)
        torch.cuda.synchronize()
        blk = sel.blk_idx.cpu().numpy()
        samp = sel.samp_idx.cpu().numpy()
        for b in range(B):
            for g in range(Hkv):
                qq = f64(q[b, g * G:(g + 1) * G])
                blocks, idx, tail = osel.select_unit(qq, f64(bm[b, g]), L, SINK, LOCAL, k)
                np.testing.assert_array_equal(blk[b, g, :len(blocks)], blocks, err_msg=str((name, pattern, k, b, g)))
                assert (blk[b, g, len(blocks):] == -1).all()
                pos = orng.sample_positions(77, b, g, 3, tail, 48)
                np.testing.assert_array_equal(samp[b, g], pos, err_msg=str((name, pattern, k, b, g)))


def test_select_wide_band_beyond_shared_memory():
    """Near-equal scores over 1012 candidates: the band exceeds the 512
    members ranked in shared memory and goes through the exact 64-bit keys in
    the workspace."""
    B, Hq, Hkv, d, L = 20, 32, 8, 128, 16384
    G = Hq // Hkv
    dev = torch.device("cuda")
    gen = torch.Generator().manual_seed(4242)
    q = torch.randn(B, Hq, d, generator=gen).to(torch.bfloat16)
    bm = _summaries("near", B, Hkv, L // 16, d, torch.bfloat16, q.float(), G, gen)
    st = sa.Stats(B, Hq, Hkv, L, d, torch.bfloat16, dev)
    st.blk_mean.copy_(bm.to(dev))
    st.mu_k.zero_()                                     # uncentred sketch
    sa.block_sketch(st, Hq)
    for k in (8, 40):
        sp = sa.SelectParams(sink=SINK, local=LOCAL, k_blocks=k)
        sel = sa.select(q.to(dev), st, sp)
        torch.cuda.synchronize()
        blk = sel.blk_idx.cpu().numpy()
        assert int(sel.n_rescored.max()) > 512
        for b, g in [(0, 0), (7, 3), (19, 7), (11, 5)]:
            blocks, _, _ = osel.select_unit(f64(q[b, g * G:(g + 1) * G]), f64(bm[b, g]), L, SINK, LOCAL, k)
            np.testing.assert_array_equal(blk[b, g], blocks)


def test_no_wait_gave_up():
    """No selection CTA in this process abandoned a bounded wait."""
    torch.cuda.synchronize()
    assert sa.wait_timeouts() == 0


# (dtype, d, Hq, Hkv, B, L): few units, so each is split over scanning CTAs
# and finished by the second kernel (keys of up to 16K candidates in shared
# memory, group top-k up to 1024 blocks, radix select beyond)
SPLIT_SHAPES = {
    "bf16_d128_g4_64k": ("bf16", 128, 8, 2, 1, 65536),
    "bf16_d128_g4_128k": ("bf16", 128, 8, 2, 1, 131072),
    "f32_d64_g2_32k": ("f32", 64, 4, 2, 2, 32768),
}


@pytest.mark.parametrize("pattern", ["random", "ties", "near"])
@pytest.mark.parametrize("name", list(SPLIT_SHAPES))
def test_select_split_units(name, pattern):
    dtype, d, Hq, Hkv, B, L = SPLIT_SHAPES[name]
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    G = Hq // Hkv
    dev = torch.device("cuda")
    gen = torch.Generator().manual_seed(zlib.crc32(("split/%s/%s" % (name, pattern)).encode()))
    q = torch.randn(B, Hq, d, generator=gen).to(dt)
    nb = L // 16
    bm = _summaries(pattern, B, Hkv, nb, d, dt, q.float(), G, gen)
    st = sa.Stats(B, Hq, Hkv, L, d, dt, dev)
    st.blk_mean.copy_(bm.to(dev))
    st.mu_k.copy_(bm.float().mean(2).to(dev))
    sa.block_sketch(st, Hq)
    qd = q.to(dev)
    n_cand = len(osel.candidate_blocks(L, SINK, LOCAL))
    for k in (8, 33, 200, 1000, n_cand - 1):
        sp = sa.SelectParams(sink=SINK, local=LOCAL, k_blocks=k, sample_b=48, sample_cap=48, seed=78, step=2)
        sel = sa.select(qd, st, sp)
        torch.cuda.synchronize()
        blk = sel.blk_idx.cpu().numpy()
        samp = sel.samp_idx.cpu().numpy()
        for b in range(B):
            for g in range(Hkv):
                qq = f64(q[b, g * G:(g + 1) * G])
                blocks, idx, tail = osel.select_unit(qq, f64(bm[b, g]), L, SINK, LOCAL, k)
                np.testing.assert_array_equal(blk[b, g, :len(blocks)], blocks, err_msg=str((name, pattern, k, b, g)))
                pos = orng.sample_positions(78, b, g, 2, tail, 48)
                np.testing.assert_array_equal(samp[b, g], pos, err_msg=str((name, pattern, k, b, g)))
