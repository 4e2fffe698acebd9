"""Host-side logic of bench.py on CPU: byte model and set geometry, clock
parsing, traffic lookup, the max-over-ranks reduction on two gloo ranks, and
the reference arm under torchrun with two ranks (rank 0 alone prints)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

import bench
import synth
from oracle import select as osel

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("L,sink,local,k", [(32768, 64, 128, 8), (2048, 16, 32, 5), (64, 16, 47, 3),
                                            (2048, 2000, 100, 5), (2048, 17, 33, 4), (4000, 64, 128, 10 ** 6)])
def test_set_geometry_matches_oracle(L, sink, local, k):
    g = bench.set_geom(L, sink, local, k)
    cand = osel.candidate_blocks(L, sink, local)
    assert g["n_cand"] == len(cand)
    assert g["kk"] == min(k, len(cand))
    idx = osel.index_set(L, sink, local, cand[: g["kk"]])
    assert g["n_i"] == len(idx) and g["n_t"] == L - len(idx)


def test_byte_model_batched():
    w = synth.WORKLOADS["batched"]
    kb = w.k_blocks_for(0.01)
    g = bench.set_geom(w.L, w.sink, w.local, kb)
    assert kb == 8 and g["n_i"] == 320
    sel = bench.select_bytes_per_unit(w, g, 2, 0)
    assert sel == 2036 * (128 + 16) + 4 * 128 * 2 + 4 * 8 + 4
    dec = bench.decode_bytes_per_unit(w, g, 2, "resa", 0)
    assert dec == 320 * 2 * 128 * 2 + 4 * 128 * 2 + 4 * 8 + 4 * 128 * 4 + 4 * (2 * 128 + 1) * 4 + 128 * 4


def test_clock_summary():
    rows = [["0", "1965", "1965", "700", "0x0", "Not Active", "Not Active", "Not Active", "Active"],
            ["0", "1800", "1965", "990", "0x4", "Not Active", "Not Active", "Not Active", "Active"],
            ["0", "1900", "1965", "995", "0x4", "Not Active", "Not Active", "Not Active", "Not Active"]]
    c = bench.summarize_clocks(rows)
    assert c["sm_mhz"] == 1900 and c["sm_max_mhz"] == 1965 and c["reasons"] == ["sw_power_cap"]
    assert bench.summarize_clocks([]) is None


def test_traffic_lookup_follows_sources(tmp_path, monkeypatch):
    got = bench.select_traffic("batched", 0.01, 256)
    if got is not None:
        assert got % 256 == 0
    monkeypatch.setattr(bench, "sources_sha1", lambda: "0" * 40)
    assert bench.select_traffic("batched", 0.01, 256) is None


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench as b
    ws, r, _ = b.dist_setup(world)
    assert ws == world and r == rank
    v = b.reduce_max(1.5 + rank)
    b.barrier()
    q.put((rank, v))
    torch.distributed.destroy_process_group()


def test_reduce_max_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: 2.5, 1: 2.5}


@pytest.mark.slow
def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "2", "--warmup", "1"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600,
                       env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle"
