#!/usr/bin/env python
"""Decode-attention benchmark: sparse decode with residual tail estimation over
a 32K bf16 GQA KV cache at a 1% read, against the in-build dense flash-decode.

    python bench.py [--gpus N --steps K --warmup W] [--impl ours|reference]

One step = one decode step of the whole batch through the hot path: block
scoring + exact top-k (sa_select, one kernel) then gather + online softmax +
residual fold + split combine (sa_decode, one kernel).  Inputs (KV cache,
prefill statistics, queries) are resident in HBM before timing; L2 is flushed
before every timed step, outside the timed events: 256 MB written, then
another 256 MB read, so that no line of the step's inputs is cached and no
dirty line of the flush is left to be written back during the step.  After
the flush the GPU spins (untimed) for ~0.1 ms so that the
step's launches are queued before its first event: the events then measure
the device time of the step, not the host's launch latency (which the e2e
figure, timed through the public API with host buffers, does include).
Prints ONE JSON line on rank 0.

--impl reference times the fp64 CPU oracle (the reference arm)
on a bounded sample of the same workload, on the host cores.
"""
import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode-attn tokens/sec & HBM GB/s (% of roofline) at 32K, 1% read, vs dense"
UNIT = "tokens/s"
FLUSH_BYTES = 256 << 20
SETTLE_CYCLES = 200_000          # GPU spin after each flush, ~0.1 ms at 2 GHz (untimed)


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="batched")
    ap.add_argument("--read", type=float, default=0.01, help="read budget (fraction of L)")
    ap.add_argument("--mode", default="resa", choices=["drop", "resa", "proxy", "sample"])
    ap.add_argument("--sample-b", type=int, default=64)
    ap.add_argument("--clt-base", type=int, default=0,
                    help="sample mode: choose b per unit by the CLT budget from this many base draws")
    ap.add_argument("--sample-cap", type=int, default=4096, help="draw capacity per unit with --clt-base")
    ap.add_argument("--budget", default="clt", choices=["clt", "clt_search", "hoeffding"],
                    help="rule for b with --clt-base")
    ap.add_argument("--eps", type=float, default=0.1)
    ap.add_argument("--delta", type=float, default=0.05)
    ap.add_argument("--queries", type=int, default=64, help="distinct decode queries cycled through")
    ap.add_argument("--dense-steps", type=int, default=50)
    ap.add_argument("--mode-steps", type=int, default=200)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-selectors", action="store_true", help="skip the alternative block scores")
    ap.add_argument("--no-multi", action="store_true", help="skip the multi-proxy (clustered) path")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--batch", type=int, default=0, help="override the batch size (profiling cases)")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# bytes the method must move (algorithmic), per unit = (sequence, KV head)

def select_bytes_per_unit(w, sg, esz, b_draws):
    """Sketch of every candidate (int8 codes + 16 bytes of scale and bounds)
    + the group's queries + outputs.  The bf16 rows of the band that is
    rescored exactly (data-dependent, typically a dozen rows) are not counted."""
    return sg["n_cand"] * (w.d + 16) + w.G * w.d * esz + 4 * sg["kk"] + 4 * b_draws + 4


def decode_bytes_per_unit(w, sg, esz, mode, b_draws):
    rows = sg["n_i"] + (b_draws if mode == "sample" else 0)
    byts = rows * 2 * w.d * esz + w.G * w.d * esz + 4 * sg["kk"] + w.G * w.d * 4
    if mode == "sample":
        byts += 4 * b_draws
    if mode == "resa":
        byts += w.G * (2 * w.d + 1) * 4 + w.d * 4       # mu_q, o_est, log_z0 per head; mu_k
    if mode == "proxy":
        byts += 2 * w.d * 4                              # sum_k, sum_v
    return byts


def scope_bytes_per_unit(w, sg, esz, mode, b_draws):
    """The method's bytes per unit and step as the scope table counts them:
    the block summaries of every candidate in the cache dtype, the group's
    queries, the exactly read K/V rows, the mode's statistics, the output
    and the chosen indices (written once, read once)."""
    byts = sg["n_cand"] * w.d * esz + w.G * w.d * esz + sg["n_i"] * 2 * w.d * esz + w.G * w.d * 4 + 8 * sg["kk"]
    if mode == "resa":
        byts += w.G * (2 * w.d * 4 + 4) + w.d * 4
    if mode == "proxy":
        byts += 2 * w.d * 4
    if mode == "sample":
        byts += b_draws * (2 * w.d * esz + 8)
    return byts


def scope_select_bytes_per_unit(w, sg, esz, b_draws):
    """The selection's share of scope_bytes_per_unit: summaries, queries,
    the chosen indices and the draws written."""
    return sg["n_cand"] * w.d * esz + w.G * w.d * esz + 4 * sg["kk"] + 4 * b_draws


def launches_per_step(w, sg, clt):
    """Kernels one sa_step launches: the selection (one kernel when every unit
    has a CTA of its own and its keys fit shared memory, else a scan and a
    finish kernel), the CLT budget's two kernels, the decode."""
    one = w.B * w.Hkv >= 148 and sg["n_cand"] <= 4096
    return (1 if one else 2) + (2 if clt else 0) + 1


def set_geom(L, sink, local, k_blocks):
    s_eff = min(sink, L)
    w_eff = min(min(local, L), L - s_eff)
    c_lo = -(-sink // 16)
    c_hi = max((L - local) // 16 if L - local > 0 else 0, c_lo)
    n_cand = c_hi - c_lo
    kk = min(k_blocks, n_cand)
    n_i = s_eff + w_eff + 16 * kk
    return {"n_cand": n_cand, "kk": kk, "n_i": n_i, "n_t": L - n_i}


# the sources k_select is compiled from (its translation unit and headers)
SELECT_SOURCES = ("kv_cache_residual_b200/csrc/sa_select.cu", "kv_cache_residual_b200/csrc/sa_select_core.cuh",
                  "kv_cache_residual_b200/csrc/sa_bulk.cuh", "kv_cache_residual_b200/csrc/sa_common.cuh",
                  "kv_cache_residual_b200/csrc/sa_internal.h", "include/sa_decode.h")


def sources_sha1():
    """sha1 over the sources of the selection kernel (name + bytes), to tell
    whether an ncu capture of it still describes the kernel being run."""
    import hashlib
    h = hashlib.sha1()
    for f in SELECT_SOURCES:
        h.update(os.path.basename(f).encode())
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()


def select_traffic(workload, read, units):
    """DRAM bytes per k_select launch from profiles/traffic.txt, scaled to
    `units`; None when absent or captured from different kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    sha = sources_sha1()
    for line in open(path):
        if line.startswith("#") or "=" not in line:
            continue
        kv = dict(tok.split("=", 1) for tok in line.split())
        if (kv.get("kernel") == "k_select" and kv.get("workload") == workload
                and abs(float(kv.get("read", "-1")) - read) < 1e-9 and kv.get("sources_sha1") == sha):
            return int(kv["bytes_per_unit"]) * units
    return None


# ---------------------------------------------------------------------------
# clocks during the timed region (nvidia-smi, read-only)

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.QUERY, "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        # nvidia-smi takes a moment to start: wait (bounded) for its first row
        # so that the sampled span covers the timed region
        t0 = time.time()
        while time.time() - t0 < 5.0 and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.05)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 9:
                rows.append(f)
        os.unlink(self.path)
        return summarize_clocks(rows)


def summarize_clocks(rows):
    if not rows:
        return None
    sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
    mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
            "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU; only timings cross ranks)

def dist_setup(n_gpus):
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return ws, rank, local


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def reduce_max(x, device=None):
    """Max of a float over ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# CPU oracle arm

def cpu_oracle_sample(w, sp_kw, mode, seconds, max_units=None, seq=0):
    """Times the fp64 oracle (select + decode of one unit = one KV head of one
    sequence) on the host, over units of one sequence, until `seconds` pass.
    Returns (units_per_s, units, threads)."""
    import numpy as np
    import torch
    from threadpoolctl import threadpool_info

    import synth
    from oracle import budget, modes, rng, select, stats

    s = synth.make_sequence(w, seq, device="cpu")
    qs = synth.make_queries(w, seq, 4, s["mu_q"], device="cpu")
    scale = 1.0 / math.sqrt(w.d)
    units = []
    for g in range(w.Hkv):
        K = s["k"][g].double().numpy()
        V = s["v"][g].double().numpy()
        st = stats.prefill_stats(s["q_ctx"][g * w.G:(g + 1) * w.G].double().numpy(), K, V, scale, w.dtype)
        units.append((g, K, V, st))
    done = 0
    t0 = time.perf_counter()
    while True:
        for g, K, V, st in units:
            step = done % qs.shape[0]
            q = qs[step, g * w.G:(g + 1) * w.G].double().numpy()
            blocks, idx, tail = select.select_unit(q, st["blk_mean"], w.L, sp_kw["sink"], sp_kw["local"],
                                                   sp_kw["k_blocks"])
            pos = None
            if mode == "sample" and sp_kw.get("clt_base", 0) > 0 and len(tail) > 0:
                # the CLT budget from the base draws, then that many draws
                base = rng.sample_positions(sp_kw["seed"], seq, g, step, tail, sp_kw["clt_base"])
                rule = {"clt": budget.clt_budget, "clt_search": budget.clt_budget_search,
                        "hoeffding": budget.hoeffding_budget}[sp_kw.get("budget", "clt")]
                b, _ = rule(q, K, V, idx, base, scale, sp_kw["eps"], sp_kw["delta"], len(tail))
                pos = rng.sample_positions(sp_kw["seed"], seq, g, step, tail, min(b, sp_kw["sample_cap"]))
            elif mode == "sample":
                pos = rng.sample_positions(sp_kw["seed"], seq, g, step, tail, sp_kw["sample_b"])
            modes.run_mode(mode, q, K, V, idx, st, scale, pos=pos)
            done += 1
            if max_units is not None and done >= max_units:
                break
        el = time.perf_counter() - t0
        if el >= seconds or (max_units is not None and done >= max_units):
            break
    threads = max([p.get("num_threads", 1) for p in threadpool_info()] or [1])
    return done / el, done, threads


def run_reference(args, w, sg, sp_kw, rank):
    if rank != 0:
        return 0
    per_step = max(1, w.Hkv)              # one step = one sequence's decode step (all KV heads)
    total = (args.warmup + args.steps) * per_step
    # bounded: the whole run stays within a few minutes
    rate, units, threads = cpu_oracle_sample(w, sp_kw, args.mode, seconds=min(120.0, 1e9), max_units=total)
    value = rate / w.Hkv
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / value, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, sg, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": "%d units (KV head x decode step) of sequence 0, mode %s, fp64 numpy" % (units, args.mode)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def workload_config(w, sg, args):
    return {"workload": "%s decode: B%d, %dq/%dkv heads, d%d, L%d, %s, %g%% read (sink %d + window %d + %d blocks of 16 = %d tokens)"
            % (w.name, w.B, w.Hq, w.Hkv, w.d, w.L, w.dtype, 100 * args.read, w.sink, w.local, sg["kk"], sg["n_i"]),
            "global_batch": w.B * args.gpus, "seq_len": w.L, "mode": args.mode, "k_blocks": sg["kk"],
            "read_tokens": sg["n_i"], "l2": "flushed before every timed step (256 MB write + 256 MB read, untimed)",
            "parallelism": "replicas (dp%d, no collective on the data path)" % args.gpus}


# ---------------------------------------------------------------------------

def main(argv=None):
    args = parse_args(argv)
    import synth
    w = synth.WORKLOADS[args.workload]
    if args.batch > 0:
        w = synth.scaled(w, B=args.batch)
    kb = w.k_blocks_for(args.read) if w.k_blocks is None else w.k_blocks
    sg = set_geom(w.L, w.sink, w.local, kb)
    sp_kw = dict(sink=w.sink, local=w.local, k_blocks=kb, sample_b=args.sample_b, seed=2024)
    if args.mode == "sample" and args.clt_base > 0:
        sp_kw.update(clt_base=args.clt_base, eps=args.eps, delta=args.delta, sample_cap=args.sample_cap,
                     budget=args.budget)
    ws, rank, local = dist_setup(args.gpus)
    if args.impl == "reference":
        rc = run_reference(args, w, sg, sp_kw, rank)
        barrier()
        return rc

    import numpy as np
    import torch

    import kv_cache_residual_b200 as sa

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    esz = 2 if w.dtype == "bf16" else 4
    nq = max(1, min(args.queries, args.steps + args.warmup))
    # weak scaling: every rank holds its own batch (sequence seeds offset by rank)
    wr = synth.scaled(w, seed=w.seed + 100_000 * rank)
    data = synth.make_batch(wr, device=dev, steps=nq)
    stats = sa.prefill_stats(data["q_ctx"], data["k"], data["v"])
    # prefill statistics (once per sequence, not part of the step): one pass
    # over the context queries and the cache
    pf_ms = []
    for r in range(4):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        sa.prefill_stats(data["q_ctx"], data["k"], data["v"], stats=stats)
        e1.record()
        torch.cuda.synchronize()
        if r > 0:
            pf_ms.append(e0.elapsed_time(e1))
    pf_bytes = (data["q_ctx"].numel() + 2 * data["k"].numel()) * data["k"].element_size()
    prefill = {"ms": statistics.mean(pf_ms), "hbm_gbs": pf_bytes / (statistics.mean(pf_ms) * 1e-3) / 1e9,
               "bytes": pf_bytes}
    # the multi-proxy path's clusters (query-geometry clustering, once per
    # sequence at prefill end): timed once, kept for the per-step timing
    clusters, qgc_ms = None, None
    if not args.no_multi:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        sa.cluster_build(data["q_ctx"][:1], data["k"][:1], data["v"][:1], n_clusters=64)     # warm-up (one sequence)
        e0.record()
        clusters = sa.cluster_build(data["q_ctx"], data["k"], data["v"], n_clusters=64)
        e1.record()
        torch.cuda.synchronize()
        qgc_ms = e0.elapsed_time(e1)
    del data["q_ctx"]
    torch.cuda.empty_cache()
    K, V, Q = data["k"], data["v"], data["q"]
    clt = args.mode == "sample" and args.clt_base > 0
    bdraw = args.sample_b if args.mode == "sample" and not clt else 0
    if clt:
        sps = [sa.SelectParams(sink=w.sink, local=w.local, k_blocks=kb, sample_b=0, sample_cap=args.sample_cap,
                               clt_base=args.clt_base, eps=args.eps, delta=args.delta, seed=2024, step=t,
                               budget=args.budget)
               for t in range(nq)]
    else:
        sps = [sa.SelectParams(sink=w.sink, local=w.local, k_blocks=kb, sample_b=bdraw, sample_cap=max(bdraw, 1),
                               seed=2024, step=t) for t in range(nq)]
    sel = sa.select(Q[0], stats, sps[0], k=K, v=V)
    out = torch.empty(w.B, w.Hq, w.d, dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

    def flush_l2():
        flush.zero_()                       # evicts the cached inputs ...
        torch.sum(flush_r)                  # ... and the dirty lines of the write
    stream = torch.cuda.current_stream()

    def step(t, mode):
        sp = sps[t % nq]
        sa.step(Q[t % nq], K, V, stats, sp, mode=mode, selection=sel, out=out)

    def timed(n, fn, n_events=3):
        """Runs fn(t, ev) n times with an L2 flush before each; returns per-step
        lists of event-pair durations (ms)."""
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_events)] for _ in range(n)]
        for t in range(n):
            flush_l2()
            torch.cuda._sleep(SETTLE_CYCLES)
            fn(t, evs[t])
        torch.cuda.synchronize()
        return [[evs[t][i].elapsed_time(evs[t][i + 1]) for i in range(n_events - 1)] for t in range(n)]

    def sparse_step(mode, sps_m=None, sel_m=None):
        """One step through sa_step (selection + decode, overlapped)."""
        sps_m = sps if sps_m is None else sps_m
        sel_m = sel if sel_m is None else sel_m

        def fn(t, ev):
            ev[0].record(stream)
            sa.step(Q[t % nq], K, V, stats, sps_m[t % nq], mode=mode, selection=sel_m, out=out)
            ev[1].record(stream)
        return fn

    def split_step(mode):
        """Selection and decode as two calls, timed separately (kernel breakdown)."""
        def fn(t, ev):
            sp = sps[t % nq]
            ev[0].record(stream)
            sa.select(Q[t % nq], stats, sp, k=K, v=V, selection=sel)
            ev[1].record(stream)
            sa.decode(Q[t % nq], K, V, stats, sel, sp, mode=mode, out=out)
            ev[2].record(stream)
        return fn

    # clocks are sampled from before the warm-up until after the dense pass,
    # so that the samples cover the timed steps whatever their number
    clocks = ClockSampler(local)
    clocks.start()
    # warm-up (untimed)
    for t in range(args.warmup):
        flush_l2()
        step(t, args.mode)
    torch.cuda.synchronize()

    barrier()
    torch.cuda.synchronize()
    per = timed(args.steps, sparse_step(args.mode), 2)
    torch.cuda.synchronize()
    barrier()
    total_ms = sum(p[0] for p in per)
    total_ms = reduce_max(total_ms, dev)
    # kernel breakdown: the same step as two calls, each bracketed by events
    timed(3, split_step(args.mode))          # warm-up: the split path's kernels load on first use
    brk = timed(min(args.steps, 500), split_step(args.mode))
    sel_ms = [p[0] for p in brk]
    dec_ms = [p[1] for p in brk]
    ms_per_step = total_ms / args.steps
    value = ws * w.B * args.steps / (total_ms / 1e3)

    b_mean = float(bdraw)
    clt_info = None
    if clt:
        # the CLT budget decides b per unit: the mean over the queries timed
        counts = []
        for t in range(nq):
            s_ = sa.select(Q[t], stats, sps[t], k=K, v=V)
            counts.append(s_.samp_count.double().mean().item())
        b_mean = statistics.mean(counts)
        clt_info = {"base": args.clt_base, "eps": args.eps, "delta": args.delta, "mean_b": b_mean,
                    "cap": args.sample_cap, "rule": args.budget}
    sel_b = select_bytes_per_unit(w, sg, esz, b_mean) * w.B * w.Hkv
    if clt:
        # the budget kernel reads I and the base draws' K and V rows
        sel_b += (sg["n_i"] + args.clt_base) * 2 * w.d * esz * w.B * w.Hkv
    dec_b = decode_bytes_per_unit(w, sg, esz, args.mode, b_mean) * w.B * w.Hkv
    peaks = {}
    pk_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pk_path):
        peaks = json.load(open(pk_path))
    peak = peaks.get("hbm_gbs")
    peak_src = "measured (MEASURED_PEAKS.json hbm_gbs)" if peak else "fallback 6650 GB/s"
    peak = peak or 6650.0
    sel_avg = statistics.mean(sel_ms)
    dec_avg = statistics.mean(dec_ms)
    sel_gbs = sel_b / (sel_avg * 1e-3) / 1e9
    dec_gbs = dec_b / (dec_avg * 1e-3) / 1e9
    step_gbs = (sel_b + dec_b) / (ms_per_step * 1e-3) / 1e9
    # the scope table's byte count (bf16 block summaries, not the int8 sketch
    # the selection actually streams)
    sv_sel = scope_select_bytes_per_unit(w, sg, esz, b_mean) * w.B * w.Hkv
    sv_step = scope_bytes_per_unit(w, sg, esz, args.mode, b_mean) * w.B * w.Hkv
    sv_sel_gbs = sv_sel / (sel_avg * 1e-3) / 1e9
    sv_step_gbs = sv_step / (ms_per_step * 1e-3) / 1e9

    # other modes (same selection kernel)
    mode_vals = {}
    for m in ("drop", "resa", "proxy", "sample"):
        sps_m, sel_m = None, None
        if m == "sample" and bdraw == 0:
            sps_m = [sa.SelectParams(sink=w.sink, local=w.local, k_blocks=kb, sample_b=args.sample_b,
                                     sample_cap=args.sample_b, seed=2024, step=t) for t in range(nq)]
            sel_m = sa.select(Q[0], stats, sps_m[0])
        fn = sparse_step(m, sps_m, sel_m)
        timed(3, fn, 2)
        pm = timed(args.mode_steps, fn, 2)
        ms = sum(p[0] for p in pm) / len(pm)
        # output error against the in-build dense attention, for one query
        o_m, _ = sa.step(Q[0], K, V, stats, (sps_m or sps)[0], mode=m)
        o_d = sa.dense_decode(Q[0], K, V)
        err = ((o_m.double() - o_d.double()).norm() / o_d.double().norm()).item()
        mode_vals[m] = {"tokens_per_s": w.B / (ms * 1e-3), "ms_per_step": ms, "rel_l2_vs_dense": err}

    # dense flash-decode reference (in-build)
    def dense_fn(t, ev):
        ev[0].record(stream)
        sa.dense_decode(Q[t % nq], K, V, out=out)
        ev[1].record(stream)
    timed(3, dense_fn, 2)
    pd = timed(args.dense_steps, dense_fn, 2)
    dense_ms = statistics.mean(p[0] for p in pd)
    clk = clocks.stop()
    dense_bytes = 2 * w.B * w.Hkv * w.L * w.d * esz + w.B * w.Hq * w.d * (esz + 4)
    dense = {"tokens_per_s": w.B / (dense_ms * 1e-3), "ms_per_step": dense_ms,
             "hbm_gbs": dense_bytes / (dense_ms * 1e-3) / 1e9,
             "frac": dense_bytes / (dense_ms * 1e-3) / 1e9 / peak}

    # end to end through the public API: pinned host q in, host output back
    e2e = None
    if not args.no_e2e:
        q_host = Q.cpu().pin_memory()
        q_dev = torch.empty_like(Q[0])
        o_host = torch.empty(w.B, w.Hq, w.d, dtype=torch.float32).pin_memory()
        # the public API's prepared call: the step's structures built once,
        # each call passes this step's query, output and step index
        prep = sa.PreparedStep(K, V, stats, sps[0], mode=args.mode, selection=sel)

        def e2e_fn(t, ev):
            ev[0].record(stream)
            q_dev.copy_(q_host[t % nq], non_blocking=True)
            ev[1].record(stream)
            prep(q_dev, out, step=sps[t % nq].step)
            ev[2].record(stream)
            o_host.copy_(out, non_blocking=True)
            ev[3].record(stream)
        timed(3, e2e_fn, 4)
        pe = timed(min(args.steps, 500), e2e_fn, 4)
        e2e_ms = reduce_max(sum(sum(p) for p in pe), dev) / len(pe)
        e2e = {"value": ws * w.B / (e2e_ms * 1e-3), "unit": UNIT, "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": int(Q[0].numel() * Q.element_size()),
               "d2h_bytes_per_step": int(out.numel() * 4),
               "h2d_us": 1e3 * statistics.mean(p[0] for p in pe),
               "step_us": 1e3 * statistics.mean(p[1] for p in pe),
               "d2h_us": 1e3 * statistics.mean(p[2] for p in pe),
               "api": "kv_cache_residual_b200.PreparedStep (sa_step), pinned host buffers"}

    # cache append (the cache growing during decode): one token per unit
    # through sa_append, written at the last row of the cache with that row's
    # own values (the cache is left as it was) into a copy of the per-unit
    # statistics; the token completes a block, so the same kernel also
    # summarises that block.  Latency-bound: a few KB per unit.
    app_st = sa.Stats.__new__(sa.Stats)
    for f in sa.Stats.FIELDS:
        t_ = getattr(stats, f)
        setattr(app_st, f, t_ if (t_ is None or f in ("blk_mean", "blk_code", "blk_meta")) else t_.clone())
    k_last = K[:, :, w.L - 1].contiguous()
    v_last = V[:, :, w.L - 1].contiguous()

    def append_fn(t, ev):
        ev[0].record(stream)
        sa.append(k_last, v_last, K, V, app_st, w.L - 1)
        ev[1].record(stream)
    timed(3, append_fn, 2)
    pa = timed(20, append_fn, 2)
    app_ms = statistics.mean(p[0] for p in pa)
    # new rows in and out, totals, mu_Q / O_Est / log_z0; the completed
    # block's 16 rows, its mean and sketch row
    app_bytes = w.B * w.Hkv * (4 * w.d * esz + 4 * w.d * 4 + w.G * (3 * w.d * 4 + 8)
                               + 17 * w.d * esz + w.d + 16)
    append = {"us_per_call": 1e3 * app_ms, "algorithmic_bytes": app_bytes,
              "note": "one token per unit completing a block (one kernel: k_append)"}
    del app_st

    # the two alternative block scores (max over the group's heads; Quest's
    # per-block key bounds): the same step with the selection ranking on them
    # (one CTA per unit scanning the bf16 means, or the min and max rows)
    selectors = None
    if not args.no_selectors:
        stats.blk_min = torch.empty_like(stats.blk_mean)
        stats.blk_max = torch.empty_like(stats.blk_mean)
        sa.block_minmax(K, 0, w.L // 16, stats, w.Hq)
        selectors = {}
        for score in ("mean_max", "quest"):
            sps_s = [dataclasses.replace(sp_, score=score) for sp_ in sps]
            fn = sparse_step(args.mode, sps_s)
            timed(3, fn, 2)
            ps_ = timed(args.mode_steps, fn, 2)
            step_ms = statistics.mean(p_[0] for p_ in ps_)

            def sel_fn(t, ev, sps_s=sps_s):
                ev[0].record(stream)
                sa.select(Q[t % nq], stats, sps_s[t % nq], k=K, v=V, selection=sel)
                ev[1].record(stream)
            timed(3, sel_fn, 2)
            pss = timed(args.mode_steps, sel_fn, 2)
            s_ms = statistics.mean(p_[0] for p_ in pss)
            rows = 2 if score == "quest" else 1
            s_bytes = (rows * sg["n_cand"] * w.d * esz + w.G * w.d * esz + 4 * sg["kk"] + 4 * b_mean) * w.B * w.Hkv
            sel_s = sa.select(Q[0], stats, sps_s[0], k=K, v=V)          # the band each unit rescored exactly
            selectors[score] = {"tokens_per_s": ws * w.B / (step_ms * 1e-3), "ms_per_step": step_ms,
                                "select_us": 1e3 * s_ms, "select_bytes": s_bytes,
                                "select_gbs": s_bytes / (s_ms * 1e-3) / 1e9,
                                "select_frac": s_bytes / (s_ms * 1e-3) / 1e9 / peak,
                                "rescored_mean": float(sel_s.n_rescored.float().mean())}
        stats.blk_min = stats.blk_max = None

    # the multi-proxy path (OpenAttention stages 02-04): ErrorGate split, the
    # QGS selector and a proxy per cluster, with the same number of tokens
    # read exactly as the block path
    multi = None
    if clusters is not None:
        budget_m = sg["n_i"]
        mout = torch.empty(w.B, w.Hq, w.d, dtype=torch.float32, device=dev)
        mread = torch.empty(w.B, w.Hkv, budget_m, dtype=torch.int32, device=dev)
        mcnt = torch.empty(w.B, w.Hkv, 64, dtype=torch.int32, device=dev)

        def multi_fn(t, ev):
            ev[0].record(stream)
            sa.multi_step(Q[t % nq], K, V, clusters, budget_m, read=mread, read_count=mcnt, out=mout)
            ev[1].record(stream)
        timed(3, multi_fn, 2)
        pm_ = timed(args.mode_steps, multi_fn, 2)
        m_ms = statistics.mean(p_[0] for p_ in pm_)
        o_m, _, _ = sa.multi_step(Q[0], K, V, clusters, budget_m)
        o_d = sa.dense_decode(Q[0], K, V)
        err = ((o_m.double() - o_d.double()).norm() / o_d.double().norm()).item()
        # per unit: codes (32 B), scale and position per token (cluster-major
        # order); the basis, the clusters' starts, counts and key /
        # squared-key / value sums; queries; the read rows; the read list and
        # counts; the output
        C_ = 64
        m_bytes = (w.L * (32 + 4 + 4) + 32 * w.d * 4 + C_ * (4 + 4 + 3 * w.d * 4) + 4 + w.G * w.d * esz
                   + budget_m * 2 * w.d * esz + budget_m * 4 + C_ * 4 + w.G * w.d * 4) * w.B * w.Hkv
        multi = {"tokens_per_s": ws * w.B / (m_ms * 1e-3), "ms_per_step": m_ms, "read_tokens": budget_m,
                 "clusters": C_, "bytes_per_step": m_bytes, "gbs": m_bytes / (m_ms * 1e-3) / 1e9,
                 "frac": m_bytes / (m_ms * 1e-3) / 1e9 / peak, "rel_l2_vs_dense": err,
                 "cluster_build_ms": qgc_ms}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu:
        rate, units, threads = cpu_oracle_sample(w, sp_kw, args.mode, args.cpu_seconds)
        cpu = {"value": rate / w.Hkv, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": "%d units (one KV head of sequence 0 at one decode step each), %.0f s, mode %s, fp64 numpy"
                         % (units, args.cpu_seconds, args.mode)}

    traffic = select_traffic(args.workload, args.read, w.B * w.Hkv)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded generator, Llama-3.1-8B layer shapes)",
            "config": dict(workload_config(w, sg, args), **({"clt": clt_info} if clt_info else {})),
            "roofline": {"bound": "hbm", "kernel": "k_select (sketch scan + certified top-k)",
                         "achieved": sv_sel_gbs, "peak": peak, "unit": "GB/s", "frac": sv_sel_gbs / peak,
                         "traffic": traffic, "bytes_per_launch": sv_sel,
                         "bytes_basis": "scope-table bytes: bf16 block summaries of every candidate + queries + indices",
                         "us_per_launch": 1e3 * sel_avg, "peak_source": peak_src,
                         "moved_bytes_per_launch": sel_b, "achieved_moved": sel_gbs, "frac_moved": sel_gbs / peak,
                         "moved_basis": "bytes the kernel streams: int8 sketch + 16 B of bounds per candidate"},
            "step_roofline": {"achieved": sv_step_gbs, "frac": sv_step_gbs / peak, "bytes_per_step": sv_step,
                              "bytes_basis": "scope-table bytes of the whole step",
                              "achieved_moved": step_gbs, "frac_moved": step_gbs / peak,
                              "moved_bytes_per_step": sel_b + dec_b,
                              "decode_gbs": dec_gbs, "decode_us": 1e3 * dec_avg, "decode_bytes": dec_b},
            "dense": dense, "speedup_vs_dense": dense_ms / ms_per_step, "modes": mode_vals,
            "kernels_us": {"k_select": 1e3 * sel_avg, "k_decode": 1e3 * dec_avg,
                           "separate_sum": 1e3 * (sel_avg + dec_avg), "step_overlapped": 1e3 * ms_per_step},
            "append": append, "prefill": prefill, "selectors": selectors, "multi_proxy": multi,
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step(w, sg, clt) * args.steps,
            "clocks": clk,
        }
        print(json.dumps(line))
    barrier()
    try:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()
    except Exception:
        pass
    return 0


if __name__ == "__main__":
    sys.exit(main())
