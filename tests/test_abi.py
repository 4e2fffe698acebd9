"""The C ABI loads, exports every symbol the header declares, sizes its
workspaces, and rejects bad arguments before launching anything.

Runs without a GPU: every call below fails argument validation, so nothing is
enqueued (the pointers passed are never dereferenced)."""
import ctypes
import os
import re

import pytest

import kv_cache_residual_b200 as sa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(sa.LIB_PATH):
        from kv_cache_residual_b200 import build
        build.build()
    return sa._lib()


def test_every_declared_symbol_is_exported(lib):
    hdr = open(os.path.join(ROOT, "include", "sa_decode.h")).read()
    declared = set(re.findall(r"^SA_API\s+[\w\s\*]+?\b(sa_\w+)\s*\(", hdr, flags=re.M))
    assert declared == set(sa.EXPORTS)
    for name in declared:
        assert hasattr(lib, name)


def _shape(**kw):
    base = dict(B=2, Hq=8, Hkv=2, d=128, L=4096, dtype=sa.SA_BF16, ld=0)
    base.update(kw)
    return sa.sa_shape(base["B"], base["Hq"], base["Hkv"], base["d"], base["L"], base["dtype"], base["ld"])


def test_workspace_sizes(lib):
    sp = sa.SelectParams(sink=64, local=128, k_blocks=8, sample_b=64, sample_cap=64).c()
    for op in range(4):
        n = lib.sa_workspace_size(ctypes.byref(_shape()), ctypes.byref(sp), op)
        assert n > 0 and n % 256 == 0
    assert lib.sa_workspace_size(ctypes.byref(_shape(d=96)), ctypes.byref(sp), 0) == 0
    assert lib.sa_workspace_size(ctypes.byref(_shape(L=100)), ctypes.byref(sp), 0) == 0
    assert lib.sa_workspace_size(None, ctypes.byref(sp), 0) == 0
    assert lib.sa_workspace_size(ctypes.byref(_shape()), None, sa.OP_SELECT) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), sa.SA_ERR_UNSUPPORTED),
    (dict(Hq=12, Hkv=4), sa.SA_ERR_UNSUPPORTED),     # G = 3
    (dict(Hq=9, Hkv=2), sa.SA_ERR_INVALID_ARG),
    (dict(L=1000), sa.SA_ERR_INVALID_ARG),          # not whole blocks and no capacity given
    (dict(L=4096, ld=4080), sa.SA_ERR_INVALID_ARG),  # capacity below the length
    (dict(L=4096, ld=4100), sa.SA_ERR_INVALID_ARG),  # capacity not whole blocks
    (dict(L=0), sa.SA_ERR_INVALID_ARG),
    (dict(B=0), sa.SA_ERR_INVALID_ARG),
    (dict(dtype=7), sa.SA_ERR_INVALID_ARG),
])
def test_bad_shapes_rejected(lib, kw, status):
    p = ctypes.c_void_p(0x10000)
    st = sa.sa_stats(*([0x10000] * 10))
    assert lib.sa_dense_decode(ctypes.byref(_shape(**kw)), p, p, p, p, 0.0, p, 1 << 30, None) == status
    assert lib.sa_prefill_stats(ctypes.byref(_shape(**kw)), p, p, p, ctypes.byref(st), 0.0, p, 1 << 30, None) == status


def test_bad_pointers_and_workspace_rejected(lib):
    sh = _shape()
    good = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10004)              # not 16-byte aligned
    assert lib.sa_dense_decode(ctypes.byref(sh), None, good, good, good, 0.0, good, 1 << 30, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_dense_decode(ctypes.byref(sh), odd, good, good, good, 0.0, good, 1 << 30, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_dense_decode(ctypes.byref(sh), good, good, good, good, -1.0, good, 1 << 30, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_dense_decode(ctypes.byref(sh), good, good, good, good, 0.0, None, 1 << 30, None) == sa.SA_ERR_WORKSPACE
    assert lib.sa_dense_decode(ctypes.byref(sh), good, good, good, good, 0.0, good, 16, None) == sa.SA_ERR_WORKSPACE
    st_bad = sa.sa_stats(0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 0x10008, 0x10000)
    assert lib.sa_prefill_stats(ctypes.byref(sh), good, good, good, ctypes.byref(st_bad), 0.0, good, 1 << 30, None) == sa.SA_ERR_INVALID_ARG


def test_select_and_decode_param_checks(lib):
    sh = _shape()
    p = ctypes.c_void_p(0x10000)
    st = sa.sa_stats(*([0x10000] * 10))
    sel = sa.sa_selection(0x10000, 0x10000, 0x10000, 0)
    bad = [
        sa.sa_select_params(-1, 128, 8, 0, 0, 0, 0.05, 0.05, 0, 0),     # negative sink
        sa.sa_select_params(64, 128, -2, 0, 0, 0, 0.05, 0.05, 0, 0),    # negative k
        sa.sa_select_params(64, 128, 8, 65, 0, 64, 0.05, 0.05, 0, 0),   # b above capacity
    ]
    for sp in bad:
        assert lib.sa_select(ctypes.byref(sh), ctypes.byref(sp), p, ctypes.byref(st), None, None,
                             ctypes.byref(sel), 0.0, p, 1 << 30, None) == sa.SA_ERR_INVALID_ARG
    clt = sa.sa_select_params(64, 128, 8, 0, 64, 512, 0.05, 0.05, 0, 0)
    # the CLT budget reads K and V
    assert lib.sa_select(ctypes.byref(sh), ctypes.byref(clt), p, ctypes.byref(st), None, None,
                         ctypes.byref(sel), 0.0, p, 1 << 30, None) == sa.SA_ERR_INVALID_ARG
    for bad_clt, status in ((sa.sa_select_params(64, 128, 8, 0, 1, 512, 0.05, 0.05, 0, 0), sa.SA_ERR_INVALID_ARG),
                            (sa.sa_select_params(64, 128, 8, 0, 300, 512, 0.05, 0.05, 0, 0), sa.SA_ERR_UNSUPPORTED),
                            (sa.sa_select_params(64, 128, 8, 0, 64, 512, 0.05, 1.0, 0, 0), sa.SA_ERR_INVALID_ARG)):
        assert lib.sa_select(ctypes.byref(sh), ctypes.byref(bad_clt), p, ctypes.byref(st), p, p,
                             ctypes.byref(sel), 0.0, p, 1 << 30, None) == status
    ok_sp = sa.sa_select_params(64, 128, 8, 0, 0, 0, 0.05, 0.05, 0, 0)
    # workspace too small
    assert lib.sa_select(ctypes.byref(sh), ctypes.byref(ok_sp), p, ctypes.byref(st), None, None,
                         ctypes.byref(sel), 0.0, p, 64, None) == sa.SA_ERR_WORKSPACE
    for mode, lam in [(9, 1.0), (1, 1.5), (1, -0.1)]:
        dp = sa.sa_decode_params(mode, lam, 0.0)
        assert lib.sa_decode(ctypes.byref(sh), ctypes.byref(dp), ctypes.byref(ok_sp), p, p, p, ctypes.byref(st),
                             ctypes.byref(sel), p, p, 1 << 30, None) == sa.SA_ERR_INVALID_ARG
    # sampling without any draw capacity
    dp = sa.sa_decode_params(sa.MODES["sample"], 1.0, 0.0)
    assert lib.sa_decode(ctypes.byref(sh), ctypes.byref(dp), ctypes.byref(ok_sp), p, p, p, ctypes.byref(st),
                         ctypes.byref(sel), p, p, 1 << 30, None) == sa.SA_ERR_INVALID_ARG
    # RESA needs its statistics
    dp = sa.sa_decode_params(sa.MODES["resa"], 1.0, 0.0)
    assert lib.sa_decode(ctypes.byref(sh), ctypes.byref(dp), ctypes.byref(ok_sp), p, p, p, None,
                         ctypes.byref(sel), p, p, 1 << 30, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_block_summaries(ctypes.byref(sh), p, 10, 5, p, p, p, p, p, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_block_summaries(ctypes.byref(sh), p, 0, 4096, p, p, p, p, p, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_block_summaries(ctypes.byref(sh), p, 0, 8, p, p, p, None, p, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_block_summaries(ctypes.byref(sh), p, 0, 8, p, p, None, p, p, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_block_summaries(ctypes.byref(sh), p, 3, 3, p, p, p, p, p, None) == sa.SA_OK   # empty range: no launch
    assert lib.sa_block_sketch(ctypes.byref(sh), p, p, 10, 5, p, p, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_block_sketch(ctypes.byref(sh), p, p, 0, 8, p, ctypes.c_void_p(0x10008), None) == sa.SA_ERR_INVALID_ARG   # misaligned
    assert lib.sa_block_sketch(ctypes.byref(sh), p, None, 0, 8, p, p, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_block_sketch(ctypes.byref(sh), p, p, 3, 3, p, p, None) == sa.SA_OK


def test_capacity_and_partial_lengths(lib):
    sp = sa.SelectParams(sink=64, local=128, k_blocks=8).c()
    # a length that is not whole blocks is valid inside a capacity that is
    for op in (sa.OP_SELECT, sa.OP_DECODE, sa.OP_DENSE):
        assert lib.sa_workspace_size(ctypes.byref(_shape(L=4100, ld=4112)), ctypes.byref(sp), op) > 0
    # but the prefill statistics cover whole blocks only
    p = ctypes.c_void_p(0x10000)
    st = sa.sa_stats(*([0x10000] * 10))
    assert lib.sa_prefill_stats(ctypes.byref(_shape(L=4100, ld=4112)), p, p, p, ctypes.byref(st), 0.0, p,
                                1 << 30, None) == sa.SA_ERR_INVALID_ARG
    # block summaries: only complete blocks of the current length
    assert lib.sa_block_summaries(ctypes.byref(_shape(L=4100, ld=4112)), p, 256, 257, p, p, p, p, p,
                                  None) == sa.SA_ERR_INVALID_ARG


def test_append_checks(lib):
    p = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)
    st = sa.sa_stats(*([0x10000] * 10))
    st_bad = sa.sa_stats(*([0x10000] * 9 + [0x10004]))
    sh = _shape(L=4096, ld=4112)
    full = _shape(L=4112, ld=4112)
    assert lib.sa_append(ctypes.byref(full), p, p, p, p, ctypes.byref(st), 0.0, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_append(ctypes.byref(_shape()), p, p, p, p, ctypes.byref(st), 0.0, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_append(ctypes.byref(sh), None, p, p, p, ctypes.byref(st), 0.0, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_append(ctypes.byref(sh), p, odd, p, p, ctypes.byref(st), 0.0, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_append(ctypes.byref(sh), p, p, p, None, ctypes.byref(st), 0.0, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_append(ctypes.byref(sh), p, p, p, p, None, 0.0, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_append(ctypes.byref(sh), p, p, p, p, ctypes.byref(st_bad), 0.0, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_append(ctypes.byref(sh), p, p, p, p, ctypes.byref(st), -1.0, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_append(ctypes.byref(_shape(L=4096, ld=4112, d=96)), p, p, p, p, ctypes.byref(st), 0.0,
                         None) == sa.SA_ERR_UNSUPPORTED


def test_status_strings(lib):
    for s in range(5):
        assert lib.sa_status_string(s)
    assert lib.sa_status_string(99) == b"unknown status"


def test_workspace_grows_with_the_clt_budget(lib):
    """The CLT budget's per-split records live in the selection workspace:
    asking for it enlarges the selection and step workspaces; sizes are
    multiples of 256 bytes and do not depend on the cache capacity beyond L."""
    plain = sa.SelectParams(sink=64, local=128, k_blocks=8, sample_b=0, sample_cap=4096).c()
    clt = sa.SelectParams(sink=64, local=128, k_blocks=8, sample_b=0, sample_cap=4096, clt_base=64,
                          eps=0.05, delta=0.05).c()
    sh = _shape(B=8, L=32768)
    for op in (sa.OP_SELECT, sa.OP_STEP):
        a = lib.sa_workspace_size(ctypes.byref(sh), ctypes.byref(plain), op)
        b = lib.sa_workspace_size(ctypes.byref(sh), ctypes.byref(clt), op)
        assert a > 0 and b > a and a % 256 == 0 and b % 256 == 0
    grown = _shape(B=8, L=32768, ld=32768 + 4096)
    for op in (sa.OP_SELECT, sa.OP_DECODE, sa.OP_DENSE):
        assert (lib.sa_workspace_size(ctypes.byref(sh), ctypes.byref(plain), op) ==
                lib.sa_workspace_size(ctypes.byref(grown), ctypes.byref(plain), op))


def test_block_score_checks(lib):
    """An unknown score, the Quest score without the block bounds, a bound
    pointer without its pair, and more candidates than the alternative scores
    hold are all rejected before anything is enqueued."""
    sh = _shape()
    p = ctypes.c_void_p(0x10000)
    st = sa.sa_stats(*([0x10000] * 10))                         # no blk_min / blk_max
    st_mm = sa.sa_stats(*([0x10000] * 12))
    st_half = sa.sa_stats(*([0x10000] * 11))                    # blk_min without blk_max
    sel = sa.sa_selection(0x10000, 0x10000, 0x10000, 0)

    def call(sp, stats, shape=sh, ws=1 << 30):
        return lib.sa_select(ctypes.byref(shape), ctypes.byref(sp), p, ctypes.byref(stats), None, None,
                             ctypes.byref(sel), 0.0, p, ws, None)

    sp = lambda score: sa.sa_select_params(64, 128, 8, 0, 0, 0, 0.05, 0.05, 0, 0, score)
    assert call(sp(3), st_mm) == sa.SA_ERR_INVALID_ARG
    assert call(sp(-1), st_mm) == sa.SA_ERR_INVALID_ARG
    assert call(sp(sa.SCORES["quest"]), st) == sa.SA_ERR_INVALID_ARG
    assert call(sp(sa.SCORES["mean_max"]), st_half) == sa.SA_ERR_INVALID_ARG
    big = _shape(B=1, L=16 * 20000)                              # 19988 candidates > 16384
    assert call(sp(sa.SCORES["mean_max"]), st_mm, shape=big) == sa.SA_ERR_UNSUPPORTED
    # accepted arguments with a workspace that is too small: the checks passed
    assert call(sp(sa.SCORES["quest"]), st_mm, ws=64) == sa.SA_ERR_WORKSPACE
    assert lib.sa_block_minmax(ctypes.byref(sh), p, 10, 5, p, p, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_block_minmax(ctypes.byref(sh), p, 0, 4096, p, p, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_block_minmax(ctypes.byref(sh), p, 0, 8, p, ctypes.c_void_p(0x10008), None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_block_minmax(ctypes.byref(sh), p, 3, 3, p, p, None) == sa.SA_OK


def test_budget_rule_checks(lib):
    sh = _shape()
    p = ctypes.c_void_p(0x10000)
    st = sa.sa_stats(*([0x10000] * 10))
    sel = sa.sa_selection(0x10000, 0x10000, 0x10000, 0)
    for rule, status in ((3, sa.SA_ERR_INVALID_ARG), (-1, sa.SA_ERR_INVALID_ARG),
                         (sa.BUDGETS["hoeffding"], sa.SA_ERR_WORKSPACE), (sa.BUDGETS["clt_search"], sa.SA_ERR_WORKSPACE)):
        sp = sa.sa_select_params(64, 128, 8, 0, 64, 512, 0.05, 0.05, 0, 0, 0, rule)
        assert lib.sa_select(ctypes.byref(sh), ctypes.byref(sp), p, ctypes.byref(st), p, p, ctypes.byref(sel), 0.0,
                             p, 64, None) == status


def test_per_head_flag_checks(lib):
    sh = _shape()
    p = ctypes.c_void_p(0x10000)
    st = sa.sa_stats(*([0x10000] * 10))
    sel = sa.sa_selection(0x10000, 0x10000, 0x10000, 0)
    for flag, status in ((2, sa.SA_ERR_INVALID_ARG), (-1, sa.SA_ERR_INVALID_ARG), (1, sa.SA_ERR_WORKSPACE)):
        sp = sa.sa_select_params(64, 128, 8, 32, 0, 32, 0.05, 0.05, 0, 0, 0, 0, flag)
        assert lib.sa_select(ctypes.byref(sh), ctypes.byref(sp), p, ctypes.byref(st), None, None, ctypes.byref(sel),
                             0.0, p, 64, None) == status
    # per-head draws need a workspace sized for G draw lists in the decode
    one = sa.sa_select_params(64, 128, 8, 32, 0, 32, 0.05, 0.05, 0, 0, 0, 0, 0)
    ph = sa.sa_select_params(64, 128, 8, 32, 0, 32, 0.05, 0.05, 0, 0, 0, 0, 1)
    assert lib.sa_workspace_size(ctypes.byref(sh), ctypes.byref(ph), sa.OP_DECODE) >= \
        lib.sa_workspace_size(ctypes.byref(sh), ctypes.byref(one), sa.OP_DECODE)


def test_cluster_entry_checks(lib):
    """sa_cluster_prep / sa_cluster_build / sa_multi_step reject a missing or
    misaligned cluster array, a cluster count outside 1..64 and an empty
    budget before launching anything; the multi-proxy workspace is
    positive and a multiple of 256 bytes."""
    sh = _shape()
    p = ctypes.c_void_p(0x10000)
    ok = sa.sa_clusters(64, *([0x10000] * 10))
    assert lib.sa_multi_step(ctypes.byref(sh), p, p, p, ctypes.byref(ok), 0, 0.0, p, p, p, p, 1 << 30,
                             None) == sa.SA_ERR_INVALID_ARG                    # budget < 1
    for bad in (sa.sa_clusters(0, *([0x10000] * 10)), sa.sa_clusters(65, *([0x10000] * 10)),
                sa.sa_clusters(64, *([0x10000] * 9 + [0])),                   # no start array
                sa.sa_clusters(64, *([0x10000] * 8 + [0, 0x10000])),          # no order array
                sa.sa_clusters(64, *([0x10008] + [0x10000] * 9))):            # misaligned basis
        assert lib.sa_cluster_prep(ctypes.byref(sh), p, p, ctypes.byref(bad), None) == sa.SA_ERR_INVALID_ARG
        assert lib.sa_cluster_build(ctypes.byref(sh), p, p, p, ctypes.byref(bad), 0, p, 1 << 30,
                                    None) == sa.SA_ERR_INVALID_ARG
        assert lib.sa_multi_step(ctypes.byref(sh), p, p, p, ctypes.byref(bad), 82, 0.0, p, p, p, p, 1 << 30,
                                 None) == sa.SA_ERR_INVALID_ARG
    none = sa.sa_select_params(0, 0, 0, 0, 0, 0, 0.0, 0.0, 0, 0)
    w = lib.sa_workspace_size(ctypes.byref(sh), ctypes.byref(none), sa.OP_MULTI)
    assert w > 0 and w % 256 == 0
    assert lib.sa_multi_step(ctypes.byref(sh), p, p, p, ctypes.byref(ok), 82, 0.0, p, p, p, p, w - 1,
                             None) == sa.SA_ERR_WORKSPACE
