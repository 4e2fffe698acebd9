"""Seeded synthetic workloads for sparse decode attention over a GQA KV cache.

This module builds inputs only: it holds none of the attention arithmetic, and
both the fp64 oracle and the CUDA path consume what it returns.

Recipe (one sequence ``b`` of a workload, generator seeded with ``seed + b``):

* typical query / key per head:  mu_Q[h] ~ N(0, I_d),  mu_K[g] ~ N(0, I_d)
* cache:    K[g, j] = mu_K[g] + sigma_k * N(0, I_d),   V[g, j] ~ N(0, I_d)
* context queries:  Q_ctx[h, t] = mu_Q[h] + N(0, I_d)
* planted heavy hitters: n_hh distinct positions per KV head, uniform over
  [0, L), get K[g, j] += 4 * qhat_g with qhat_g the unit vector along
  sum_{h in group g} mu_Q[h]
* decode queries: q_t[h] = mu_Q[h] + N(0, I_d), drawn from a generator seeded
  by (seed + b, t)
* everything is rounded to the workload dtype (bf16 RNE, or kept fp32) after
  planting.

The shapes follow a Llama-3.1-8B attention layer (32 query / 8 KV heads,
d = 128, bf16), the model the RESA, vAttention and OpenAttention pages
evaluate on; the pages' benchmark datasets (RULER, LongBench, AIME) are not
used: these seeded tensors stand in for them.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Tuple

import torch

BLOCK = 16


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    L: int
    dtype: str            # "f32" or "bf16": KV cache, context and decode queries
    steps: int            # decode steps (fresh query each)
    sink: int             # attention-sink tokens read exactly
    local: int            # local-window tokens read exactly
    read_fracs: Tuple[float, ...]   # read budgets (fraction of L read exactly)
    n_hh: int             # planted heavy hitters per KV head
    sigma_k: float        # key noise around mu_K
    seed: int
    k_blocks: Optional[int] = None  # explicit top-block count (overrides read_fracs)
    sample_b: int = 64    # draws for the sampling estimator (0 = CLT budget)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def k_blocks_for(self, rho: float) -> int:
        """Top-block count for a read budget rho: floor((rho*L - sink - local)/16)."""
        return max(0, int(math.floor((rho * self.L - self.sink - self.local) / BLOCK + 1e-9)))

    def budgets(self):
        """[(label, k_blocks)] for this workload."""
        if self.k_blocks is not None:
            return [("k%d" % self.k_blocks, self.k_blocks)]
        return [("%g%%" % (100 * r), self.k_blocks_for(r)) for r in self.read_fracs]


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", B=1, Hq=4, Hkv=1, d=64, L=2048, dtype="f32", steps=8,
                     sink=16, local=32, read_fracs=(), n_hh=8, sigma_k=1.0, seed=0,
                     k_blocks=5, sample_b=64),
    "llama": Workload("llama", B=1, Hq=32, Hkv=8, d=128, L=32768, dtype="bf16", steps=16,
                      sink=64, local=128, read_fracs=(0.01, 0.03), n_hh=64, sigma_k=1.0,
                      seed=1),
    "batched": Workload("batched", B=32, Hq=32, Hkv=8, d=128, L=32768, dtype="bf16",
                        steps=64, sink=64, local=128, read_fracs=(0.01,), n_hh=64,
                        sigma_k=1.0, seed=1000),
    "long": Workload("long", B=4, Hq=32, Hkv=8, d=128, L=131072, dtype="bf16", steps=32,
                     sink=64, local=128, read_fracs=(0.005, 0.02), n_hh=64, sigma_k=1.0,
                     seed=2000),
    "flat": Workload("flat", B=8, Hq=32, Hkv=8, d=128, L=32768, dtype="bf16", steps=16,
                     sink=64, local=128, read_fracs=(0.01, 0.02, 0.05, 0.10), n_hh=0,
                     sigma_k=0.25, seed=3000, sample_b=0),
}


def scaled(w: Workload, **kw) -> Workload:
    """The same recipe with some fields replaced (smaller parity cases)."""
    return dataclasses.replace(w, **kw)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return g


def _query_seed(seq_seed: int, step: int) -> int:
    return (seq_seed + 1) * 1_000_003 + 7919 * (step + 1)


def make_sequence(w: Workload, b: int, device="cpu", with_qctx: bool = True):
    """One sequence: dict with k, v [Hkv, L, d], q_ctx [Hq, L, d] (workload dtype),
    mu_q [Hq, d] and mu_k [Hkv, d] (fp32, the generator's means, for diagnostics)
    and hh [Hkv, n_hh] (planted positions)."""
    dev = torch.device(device)
    g = _gen(dev, w.seed + b)
    f32 = torch.float32
    mu_q = torch.randn(w.Hq, w.d, generator=g, device=dev, dtype=f32)
    mu_k = torch.randn(w.Hkv, w.d, generator=g, device=dev, dtype=f32)
    k = mu_k[:, None, :] + w.sigma_k * torch.randn(w.Hkv, w.L, w.d, generator=g, device=dev, dtype=f32)
    v = torch.randn(w.Hkv, w.L, w.d, generator=g, device=dev, dtype=f32)
    hh = torch.empty(w.Hkv, w.n_hh, dtype=torch.long, device=dev)
    if w.n_hh > 0:
        qsum = mu_q.view(w.Hkv, w.G, w.d).sum(1)
        qhat = qsum / qsum.norm(dim=-1, keepdim=True)
        for gi in range(w.Hkv):
            pos = torch.randperm(w.L, generator=g, device=dev)[: w.n_hh]
            hh[gi] = pos
            k[gi, pos] += 4.0 * qhat[gi]
    out = {"k": k.to(w.torch_dtype), "v": v.to(w.torch_dtype), "mu_q": mu_q, "mu_k": mu_k, "hh": hh}
    del k, v
    if with_qctx:
        q_ctx = torch.empty(w.Hq, w.L, w.d, dtype=w.torch_dtype, device=dev)
        for h in range(w.Hq):  # one head at a time keeps the fp32 temporary small
            q_ctx[h] = (mu_q[h][None, :] + torch.randn(w.L, w.d, generator=g, device=dev, dtype=f32)).to(w.torch_dtype)
        out["q_ctx"] = q_ctx
    return out


def make_queries(w: Workload, b: int, steps: int, mu_q: torch.Tensor, device="cpu", first_step: int = 0):
    """Decode queries for steps [first_step, first_step+steps): [steps, Hq, d]."""
    dev = torch.device(device)
    out = torch.empty(steps, w.Hq, w.d, dtype=w.torch_dtype, device=dev)
    for i in range(steps):
        g = _gen(dev, _query_seed(w.seed + b, first_step + i))
        out[i] = (mu_q.to(dev) + torch.randn(w.Hq, w.d, generator=g, device=dev, dtype=torch.float32)).to(w.torch_dtype)
    return out


def make_batch(w: Workload, device="cpu", steps: Optional[int] = None, with_qctx: bool = True):
    """Whole batch: k, v [B, Hkv, L, d]; q_ctx [B, Hq, L, d]; queries [steps, B, Hq, d]."""
    steps = w.steps if steps is None else steps
    dev = torch.device(device)
    K = torch.empty(w.B, w.Hkv, w.L, w.d, dtype=w.torch_dtype, device=dev)
    V = torch.empty_like(K)
    Qc = torch.empty(w.B, w.Hq, w.L, w.d, dtype=w.torch_dtype, device=dev) if with_qctx else None
    Q = torch.empty(steps, w.B, w.Hq, w.d, dtype=w.torch_dtype, device=dev)
    mus = []
    for b in range(w.B):
        s = make_sequence(w, b, dev, with_qctx=with_qctx)
        K[b] = s["k"]
        V[b] = s["v"]
        if with_qctx:
            Qc[b] = s["q_ctx"]
        Q[:, b] = make_queries(w, b, steps, s["mu_q"], dev)
        mus.append(s["mu_q"])
        del s
    return {"k": K, "v": V, "q_ctx": Qc, "q": Q, "mu_q": torch.stack(mus)}
