"""Helpers for the GPU-vs-oracle parity tests: run the CUDA path through the
binding and the fp64 oracle on the same synthetic unit, and compare."""
import math

import numpy as np
import torch

from oracle import modes as omodes
from oracle import rng as orng
from oracle import select as osel
from oracle import stats as ostats

REL_L2_OUT = 2e-3       # output bar (fp32 kernels vs fp64 oracle)


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


class OracleUnit:
    """fp64 oracle state for unit (b, g) of a batch held on the GPU."""

    def __init__(self, data, b, g, G, dtype, scale=None):
        self.b, self.g, self.G = b, g, G
        self.k = f64(data["k"][b, g])
        self.v = f64(data["v"][b, g])
        self.L, self.d = self.k.shape
        self.scale = 1.0 / math.sqrt(self.d) if scale is None else scale
        qctx = f64(data["q_ctx"][b, g * G:(g + 1) * G])
        self.st = ostats.prefill_stats(qctx, self.k, self.v, self.scale, dtype)

    def q(self, q_step):
        return f64(q_step[self.b, self.g * self.G:(self.g + 1) * self.G])

    def select(self, q, sp):
        return osel.select_unit(q, self.st["blk_mean"], self.L, sp.sink, sp.local, sp.k_blocks)

    def draws(self, tail, sp, n):
        return orng.sample_positions(sp.seed, self.b, self.g, sp.step, tail, n)

    def out(self, mode, q, idx, pos=None, lam=1.0):
        return omodes.run_mode(mode, q, self.k, self.v, idx, self.st, self.scale, pos=pos, lam=lam)
