"""GPU checks of the scan sketch (int8 codes of the block summaries minus
the unit's typical key, with per-row scale and error bounds): scales and
codes exactly as their definition states, bounds never below the exact norms
and tight."""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import kv_cache_residual_b200 as sa

pytestmark = pytest.mark.gpu


def _reference(kbar, centre):
    """kbar [rows, d] float64 holding bf16 / fp32 values, centre [rows, d]
    fp32 values -> s, codes, ||t - s code||_2 and ||s code||_2 with
    t = kbar - centre (rational arithmetic: exact, then rounded)."""
    x = kbar - centre                     # as the kernel forms it (fp64)
    amax = np.abs(x).max(axis=1).astype(np.float32)
    s = (amax / np.float32(127.0)).astype(np.float32)
    s64 = s.astype(np.float64)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        c = np.where(s64 > 0, np.clip(np.rint(x / s64), -127, 127), 0.0)
    def exact_norm(krow, crow, codes, sv):
        sq = sum((Fraction(float(a)) - Fraction(float(b)) - Fraction(float(sv)) * int(cv)) ** 2
                 for a, b, cv in zip(krow, crow, codes))
        return math.sqrt(sq)                 # within half an ulp of the exact norm

    r = np.array([exact_norm(kr, cr, cc, sv) for kr, cr, cc, sv in zip(kbar, centre, c, s)])
    k = np.sqrt(((s64 * c) ** 2).sum(axis=1))
    return s, c.astype(np.int8), r, k


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.bfloat16, 64), (torch.float32, 128),
                                     (torch.float32, 64)])
def test_sketch_matches_definition(dtype, d):
    B, Hq, Hkv, L = 3, 8, 2, 1024
    gen = torch.Generator().manual_seed(d + (1 if dtype == torch.float32 else 0))
    nb = L // 16
    m = torch.randn(B, Hkv, nb, d, generator=gen)
    m[0, 0, 3] = 0.0                                          # all-zero row
    m[0, 1, 5] *= 1e-30                                       # tiny row
    m[1, 0, 7] *= 1e30 if dtype == torch.float32 else 1e20    # huge row
    m[2, 1, 9, :] = 0.0
    m[2, 1, 9, 17] = -3.0                                     # one non-zero element
    m = m.to(dtype)
    dev = torch.device("cuda")
    st = sa.Stats(B, Hq, Hkv, L, d, dtype, dev)
    centre = (0.5 * torch.randn(B, Hkv, d, generator=gen)).float()
    centre[0, 0] = 0.0                                        # uncentred unit
    st.blk_mean.copy_(m.to(dev))
    st.mu_k.copy_(centre.to(dev))
    st.blk_code.fill_(99)
    st.blk_meta.fill_(-1.0)
    sa.block_sketch(st, Hq, 1, nb)                            # row 0 of each unit left untouched
    torch.cuda.synchronize()
    code = st.blk_code.cpu().numpy()
    meta = st.blk_meta.cpu().numpy()
    assert (code[:, :, 0] == 99).all() and (meta[:, :, 0] == -1.0).all()
    x = m.double().numpy()[:, :, 1:].reshape(-1, d)
    cen = np.broadcast_to(centre.double().numpy()[:, :, None, :], (B, Hkv, nb - 1, d)).reshape(-1, d)
    s, c, r, k = _reference(x, cen)
    got_c = code[:, :, 1:].reshape(-1, d)
    got_m = meta[:, :, 1:].reshape(-1, 4)
    np.testing.assert_array_equal(got_m[:, 0], s)
    np.testing.assert_array_equal(got_c, c)
    assert (got_m[:, 3] == 0).all()
    for got, exact in ((got_m[:, 1].astype(np.float64), r), (got_m[:, 2].astype(np.float64), k)):
        assert (got >= exact).all()
        assert (got <= exact * (1 + 2.0 ** -20) + 1e-300).all()


def test_prefill_writes_the_sketch_of_its_means():
    import synth
    w = synth.scaled(synth.WORKLOADS["llama"], B=2, Hq=8, Hkv=2, L=2048, n_hh=8, seed=5)
    dev = torch.device("cuda")
    data = synth.make_batch(w, device=dev, steps=1)
    st = sa.prefill_stats(data["q_ctx"], data["k"], data["v"])
    code, meta = st.blk_code.clone(), st.blk_meta.clone()
    sa.block_sketch(st, w.Hq)
    torch.cuda.synchronize()
    assert torch.equal(code, st.blk_code) and torch.equal(meta, st.blk_meta)
