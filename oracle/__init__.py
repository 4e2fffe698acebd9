"""fp64 CPU oracle for sparse single-token decode attention with residual tail
estimation (RESA rank-1 prior, count-aware mean proxy, uniform tail sampling).

TEST INFRASTRUCTURE ONLY.  Only tests/, ``__graft_entry__.smoke()`` and the
cpu_baseline / reference arm of ``bench.py`` import this package.  The product
path (``kv_cache_residual_b200``) never imports it, and it never imports the
product path; the two share no code.  The seeded input generator lives in
``synth`` and holds none of the method's arithmetic.

Everything works on ONE unit u = (sequence b, KV head g): keys and values
K, V in R^{L x d}, the G query heads of the group, all as float64 arrays
holding the exact values of the cache (bf16 or fp32 upcast).

Sources (pages, by title and section):

* RESA: Bringing Back What Sparse Attention Ignores with Residual Estimation
  - Method, key design 1 "Prior Estimator": rank-1 logit prior, bias term,
    O_Est computed once at prefill end as one extra query.
  - Method, key design 2 "Online Aggregator": Z, Z', alpha, beta rescale and
    the delta-merge equation for O_RESA; lambda prior weight; log-sum-exp.
* vAttention: Verified Sparse Attention via Sampling
  - Method, overall framework: I_f = sink + local + top-k; uniform sampling of
    the residual.
  - Key design 1: the probability-weighted numerator/denominator (paper eq. 3)
    with samples reweighted by n_s / |I_dyn|.
  - Key design 2: CLT sampling-budget lemma; key design 3: Lemma 4.2.
* OpenAttention: One Percent Is Enough with Tail Proxies
  - Abstract and method stage 04: the count-aware mean proxy, one virtual
    token with logit zbar + log n and value = the tail mean.
  - Method overview stages 01-04 (openattn.py): query-geometry clustering,
    ErrorGate's budget split, the QGS int8 selector and one proxy per cluster.

Parity status of each function is stated in its docstring; the pins live in
tests/test_oracle_*.py.
"""
from . import numerics, rng, select, stats, modes, budget, openattn  # noqa: F401
