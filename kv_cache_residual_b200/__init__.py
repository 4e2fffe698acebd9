"""Python binding of libsa_b200.so: sparse single-token decode attention over
a GQA KV cache with residual tail estimation, on NVIDIA B200 (sm_100a).

Argument marshalling only: every step runs in the library's CUDA kernels.
PyTorch provides device memory and the current stream.  There is no CPU
fallback: if the shared library is missing, importing the ops raises.

Layouts: k, v [B, Hkv, L, d]; q_ctx [B, Hq, L, d]; q [B, Hq, d]; bf16 or fp32
(one dtype for all); outputs fp32 [B, Hq, d].

    stats = prefill_stats(q_ctx, k, v)
    sp = SelectParams(sink=64, local=128, k_blocks=8, sample_b=64, sample_cap=64, seed=1, step=t)
    sel = select(q, stats, sp)
    o = decode(q, k, v, stats, sel, sp, mode="resa")
"""
import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsa_b200.so")

SA_OK, SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_WORKSPACE, SA_ERR_CUDA = range(5)
SA_F32, SA_BF16 = 0, 1
MODES = {"drop": 0, "resa": 1, "proxy": 2, "sample": 3}
SCORES = {"mean_sum": 0, "mean_max": 1, "quest": 2}
BUDGETS = {"clt": 0, "clt_search": 1, "hoeffding": 2}
OP_PREFILL, OP_SELECT, OP_DECODE, OP_DENSE, OP_STEP, OP_MULTI, OP_CLUSTER = range(7)


class SAError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__("%s: %s (status %d)" % (what, _lib().sa_status_string(status).decode(), status))


class sa_shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("d", ctypes.c_int),
                ("L", ctypes.c_int), ("dtype", ctypes.c_int), ("ld", ctypes.c_int)]


class sa_stats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("mu_q", "o_est", "log_z0", "mu_k", "sum_k", "sum_v", "blk_mean", "kbar_absmax", "blk_code",
                 "blk_meta", "blk_min", "blk_max")]


class sa_select_params(ctypes.Structure):
    _fields_ = [("sink", ctypes.c_int), ("local", ctypes.c_int), ("k_blocks", ctypes.c_int),
                ("sample_b", ctypes.c_int), ("clt_base", ctypes.c_int), ("sample_cap", ctypes.c_int),
                ("eps", ctypes.c_float), ("delta", ctypes.c_float), ("seed", ctypes.c_uint64),
                ("step", ctypes.c_int), ("score", ctypes.c_int), ("budget", ctypes.c_int),
                ("per_head", ctypes.c_int)]


class sa_selection(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("blk_idx", "samp_idx", "samp_count", "n_rescored")]


class sa_clusters(ctypes.Structure):
    _fields_ = [("n_clusters", ctypes.c_int)] + [(n, ctypes.c_void_p) for n in
                                                  ("basis", "assign", "codes", "scales", "count", "sum_k", "sum_v",
                                                   "sum_k2", "order", "start")]


class sa_decode_params(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int), ("lam", ctypes.c_float), ("scale", ctypes.c_float)]


EXPORTS = ("sa_workspace_size", "sa_prefill_stats", "sa_block_summaries", "sa_block_sketch", "sa_block_minmax",
           "sa_select",
           "sa_select_noalloc",
           "sa_decode", "sa_step", "sa_dense_decode", "sa_append", "sa_wait_timeouts", "sa_cluster_prep", "sa_cluster_build",
           "sa_multi_step",
           "sa_status_string")

_LIB = None


def _lib():
    """Load the shared library (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libsa_b200.so not built: run `python -m kv_cache_residual_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        sh, sp = ctypes.POINTER(sa_shape), ctypes.POINTER(sa_select_params)
        st, sel, dp = ctypes.POINTER(sa_stats), ctypes.POINTER(sa_selection), ctypes.POINTER(sa_decode_params)
        lib.sa_workspace_size.argtypes = [sh, sp, I]
        lib.sa_workspace_size.restype = S
        lib.sa_prefill_stats.argtypes = [sh, P, P, P, st, F, P, S, P]
        lib.sa_block_summaries.argtypes = [sh, P, I, I, P, P, P, P, P, P]
        lib.sa_block_sketch.argtypes = [sh, P, P, I, I, P, P, P]
        lib.sa_block_minmax.argtypes = [sh, P, I, I, P, P, P]
        lib.sa_select.argtypes = [sh, sp, P, st, P, P, sel, F, P, S, P]
        lib.sa_select_noalloc.argtypes = [sh, sp, P, st, P, P, sel, F, P]
        lib.sa_decode.argtypes = [sh, dp, sp, P, P, P, st, sel, P, P, S, P]
        lib.sa_step.argtypes = [sh, dp, sp, P, P, P, st, sel, P, P, S, P]
        lib.sa_dense_decode.argtypes = [sh, P, P, P, P, F, P, S, P]
        lib.sa_append.argtypes = [sh, P, P, P, P, st, F, P]
        cl = ctypes.POINTER(sa_clusters)
        lib.sa_cluster_prep.argtypes = [sh, P, P, cl, P]
        lib.sa_cluster_build.argtypes = [sh, P, P, P, cl, I, P, S, P]
        lib.sa_multi_step.argtypes = [sh, P, P, P, cl, I, F, P, P, P, P, S, P]
        lib.sa_wait_timeouts.argtypes = [ctypes.POINTER(ctypes.c_uint)]
        lib.sa_wait_timeouts.restype = I
        lib.sa_status_string.argtypes = [I]
        lib.sa_status_string.restype = ctypes.c_char_p
        for f in ("sa_cluster_prep", "sa_cluster_build", "sa_multi_step",
                  "sa_prefill_stats", "sa_block_summaries", "sa_block_sketch", "sa_block_minmax", "sa_select", "sa_select_noalloc", "sa_decode", "sa_step",
                  "sa_dense_decode", "sa_append"):
            getattr(lib, f).restype = I
        _LIB = lib
    return _LIB


def _check(status, what):
    if status != SA_OK:
        raise SAError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return SA_BF16
    if t.dtype == torch.float32:
        return SA_F32
    raise TypeError("cache dtype must be bfloat16 or float32, got %s" % t.dtype)


def make_shape(k, Hq, length=None):
    """Shape of a cache tensor k [B, Hkv, ld, d] holding `length` valid tokens
    per unit (default: all ld)."""
    B, Hkv, ld, d = k.shape
    return sa_shape(B, Hq, Hkv, d, ld if length is None else int(length), _dtype_code(k), ld)


@dataclass
class SelectParams:
    sink: int = 64
    local: int = 128
    k_blocks: int = 8
    sample_b: int = 0
    sample_cap: int = 0
    clt_base: int = 0
    eps: float = 0.05
    delta: float = 0.05
    seed: int = 0
    step: int = 0
    score: str = "mean_sum"          # block score: "mean_sum", "mean_max" or "quest"
    budget: str = "clt"              # with clt_base > 0: "clt", "clt_search" or "hoeffding"
    per_head: bool = False           # draws and budget per query head (not per KV head)

    def c(self):
        return sa_select_params(self.sink, self.local, self.k_blocks, self.sample_b, self.clt_base,
                                max(self.sample_cap, self.sample_b), self.eps, self.delta,
                                self.seed & ((1 << 64) - 1), self.step, SCORES[self.score],
                                BUDGETS[self.budget], int(bool(self.per_head)))


class Stats:
    """Prefill-end statistics (caller-owned device tensors)."""

    FIELDS = ("mu_q", "o_est", "log_z0", "mu_k", "sum_k", "sum_v", "blk_mean", "kbar_absmax", "blk_code",
              "blk_meta", "blk_min", "blk_max")

    def __init__(self, B, Hq, Hkv, L, d, dtype, device, minmax=False):
        f = dict(dtype=torch.float32, device=device)
        self.mu_q = torch.empty(B, Hq, d, **f)
        self.o_est = torch.empty(B, Hq, d, **f)
        self.log_z0 = torch.empty(B, Hq, **f)
        self.mu_k = torch.empty(B, Hkv, d, **f)
        self.sum_k = torch.empty(B, Hkv, d, **f)
        self.sum_v = torch.empty(B, Hkv, d, **f)
        self.blk_mean = torch.empty(B, Hkv, L // 16, d, dtype=dtype, device=device)
        self.kbar_absmax = torch.zeros(B, Hkv, **f)
        # scan sketch of blk_mean (int8 codes + {scale, residual norm, norm, 0})
        self.blk_code = torch.empty(B, Hkv, L // 16, d, dtype=torch.int8, device=device)
        self.blk_meta = torch.empty(B, Hkv, L // 16, 4, **f)
        # per-block key minimum and maximum (the "quest" block score), on request
        self.blk_min = torch.empty(B, Hkv, L // 16, d, dtype=dtype, device=device) if minmax else None
        self.blk_max = torch.empty(B, Hkv, L // 16, d, dtype=dtype, device=device) if minmax else None

    def c(self):
        return sa_stats(*[None if self.__dict__.get(n) is None else self.__dict__[n].data_ptr()
                          for n in self.FIELDS])


class Selection:
    """Output of select(): chosen blocks per unit and tail draws per unit (or,
    with per-head sampling, per query head: draw_rows = Hq)."""

    def __init__(self, B, Hkv, k_blocks, sample_cap, device, draw_rows=None):
        i = dict(dtype=torch.int32, device=device)
        rows = Hkv if draw_rows is None else draw_rows
        self.blk_idx = torch.empty(B, Hkv, max(k_blocks, 1), **i)
        self.samp_idx = torch.empty(B, rows, max(sample_cap, 1), **i)
        self.samp_count = torch.zeros(B, rows, **i)
        self.n_rescored = torch.zeros(B, Hkv, **i)

    def c(self):
        return sa_selection(self.blk_idx.data_ptr(), self.samp_idx.data_ptr(), self.samp_count.data_ptr(),
                            self.n_rescored.data_ptr())


class Clusters:
    """The multi-proxy state of a cache (caller-owned device tensors, layouts
    of sa_clusters in sa_decode.h)."""

    FIELDS = ("basis", "assign", "codes", "scales", "count", "sum_k", "sum_v", "sum_k2", "order", "start")

    def __init__(self, B, Hkv, ld, d, n_clusters, device):
        f = dict(dtype=torch.float32, device=device)
        self.n_clusters = int(n_clusters)
        self.basis = torch.zeros(B, Hkv, 32, d, **f)
        self.assign = torch.zeros(B, Hkv, ld, dtype=torch.uint8, device=device)
        self.codes = torch.zeros(B, Hkv, ld, 32, dtype=torch.int8, device=device)
        self.scales = torch.zeros(B, Hkv, ld, **f)
        self.count = torch.zeros(B, Hkv, n_clusters, dtype=torch.int32, device=device)
        self.sum_k = torch.zeros(B, Hkv, n_clusters, d, **f)
        self.sum_v = torch.zeros(B, Hkv, n_clusters, d, **f)
        self.sum_k2 = torch.zeros(B, Hkv, n_clusters, d, **f)
        self.order = torch.zeros(B, Hkv, ld, dtype=torch.int32, device=device)
        self.start = torch.zeros(B, Hkv, n_clusters + 1, dtype=torch.int32, device=device)

    def c(self):
        return sa_clusters(self.n_clusters, *[getattr(self, n).data_ptr() for n in self.FIELDS])


def cluster_prep(k, v, clusters, Hq, length=None, stream=None):
    """Codes, scales, counts and sums of `clusters` from its basis and
    assignment over the first `length` tokens (see sa_cluster_prep)."""
    shape = make_shape(k, Hq, length)
    c = clusters.c()
    _check(_lib().sa_cluster_prep(ctypes.byref(shape), _ptr(k), _ptr(v), ctypes.byref(c), _stream(stream)),
           "sa_cluster_prep")


def cluster_build(q_ctx, k, v, n_clusters=64, clusters=None, basis_given=False, length=None, stream=None):
    """Query-geometry clustering of the cache (see sa_cluster_build): basis
    (unless given in `clusters`), assignment, codes and sums.  Returns the
    Clusters."""
    B, Hkv, ld, d = k.shape
    Hq = q_ctx.shape[1] if q_ctx is not None else None
    if Hq is None:
        raise ValueError("q_ctx gives the number of query heads")
    shape = make_shape(k, Hq, length if length is not None else q_ctx.shape[2])
    if clusters is None:
        clusters = Clusters(B, Hkv, ld, d, n_clusters, k.device)
    ws = workspace(shape, None, OP_CLUSTER, k.device)
    c = clusters.c()
    _check(_lib().sa_cluster_build(ctypes.byref(shape), _ptr(q_ctx), _ptr(k), _ptr(v), ctypes.byref(c),
                                   int(bool(basis_given)), _ptr(ws), ws.numel(), _stream(stream)),
           "sa_cluster_build")
    return clusters


def multi_step(q, k, v, clusters, budget, scale=0.0, read=None, read_count=None, out=None, length=None,
               stream=None):
    """One multi-proxy decode step (see sa_multi_step).  Returns (out, read,
    read_count)."""
    B, Hq, d = q.shape
    shape = make_shape(k, Hq, length)
    Hkv = shape.Hkv
    dev = q.device
    if read is None:
        read = torch.empty(B, Hkv, int(budget), dtype=torch.int32, device=dev)
    if read_count is None:
        read_count = torch.empty(B, Hkv, clusters.n_clusters, dtype=torch.int32, device=dev)
    if out is None:
        out = torch.empty(B, Hq, d, dtype=torch.float32, device=dev)
    ws = workspace(shape, None, OP_MULTI, dev)
    c = clusters.c()
    _check(_lib().sa_multi_step(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), ctypes.byref(c), int(budget),
                                float(scale), _ptr(read), _ptr(read_count), _ptr(out), _ptr(ws), ws.numel(),
                                _stream(stream)), "sa_multi_step")
    return out, read, read_count


_WS = {}


def workspace(shape, params, op, device):
    """Zero-filled scratch for one op, cached per (device, op, shape, params)."""
    lib = _lib()
    n = lib.sa_workspace_size(ctypes.byref(shape), ctypes.byref(params) if params is not None else None, op)
    if n == 0:
        raise SAError(SA_ERR_INVALID_ARG, "sa_workspace_size")
    key = (str(device), op, n)
    ws = _WS.get(key)
    if ws is None:
        ws = torch.zeros(n, dtype=torch.uint8, device=device)
        _WS[key] = ws
    return ws


def prefill_stats(q_ctx, k, v, stats=None, scale=0.0, stream=None, minmax=False):
    """Statistics of the first L = q_ctx.shape[2] tokens of a cache k, v
    [B, Hkv, ld, d] (ld >= L: room for appended tokens); minmax: also the
    per-block key bounds the "quest" block score ranks on."""
    B, Hkv, ld, d = k.shape
    Hq, L = q_ctx.shape[1], q_ctx.shape[2]
    shape = make_shape(k, Hq, L)
    if stats is None:
        stats = Stats(B, Hq, Hkv, ld, d, k.dtype, k.device, minmax=minmax)
    ws = workspace(shape, None, OP_PREFILL, k.device)
    st = stats.c()
    _check(_lib().sa_prefill_stats(ctypes.byref(shape), _ptr(q_ctx), _ptr(k), _ptr(v), ctypes.byref(st),
                                   float(scale), _ptr(ws), ws.numel(), _stream(stream)), "sa_prefill_stats")
    return stats


def block_summaries(k, blk_begin, blk_end, stats, Hq, length=None, stream=None):
    shape = make_shape(k, Hq, length)
    _check(_lib().sa_block_summaries(ctypes.byref(shape), _ptr(k), int(blk_begin), int(blk_end),
                                     _ptr(stats.blk_mean), _ptr(stats.kbar_absmax), _ptr(stats.mu_k),
                                     _ptr(stats.blk_code), _ptr(stats.blk_meta), _stream(stream)),
           "sa_block_summaries")


def block_minmax(k, blk_begin, blk_end, stats, Hq, length=None, stream=None):
    """Key minimum and maximum of blocks [blk_begin, blk_end) of every unit into
    stats.blk_min / stats.blk_max (see sa_block_minmax)."""
    shape = make_shape(k, Hq, length)
    _check(_lib().sa_block_minmax(ctypes.byref(shape), _ptr(k), int(blk_begin), int(blk_end), _ptr(stats.blk_min),
                                  _ptr(stats.blk_max), _stream(stream)), "sa_block_minmax")


def block_sketch(stats, Hq, blk_begin=0, blk_end=None, stream=None):
    """Rebuilds stats.blk_code / blk_meta from stats.blk_mean relative to
    stats.mu_k (blocks [blk_begin, blk_end) of every unit), for block means or
    a mu_k written by hand."""
    B, Hkv, nb, d = stats.blk_mean.shape
    shape = sa_shape(B, Hq, Hkv, d, nb * 16, _dtype_code(stats.blk_mean))
    blk_end = nb if blk_end is None else blk_end
    _check(_lib().sa_block_sketch(ctypes.byref(shape), _ptr(stats.blk_mean), _ptr(stats.mu_k), int(blk_begin),
                                  int(blk_end),
                                  _ptr(stats.blk_code), _ptr(stats.blk_meta), _stream(stream)),
           "sa_block_sketch")


def select(q, stats, params, k=None, v=None, selection=None, scale=0.0, length=None, stream=None):
    B, Hq, d = q.shape
    Hkv, ld = stats.blk_mean.shape[1], stats.blk_mean.shape[2] * 16
    shape = sa_shape(B, Hq, Hkv, d, ld if length is None else int(length), _dtype_code(q), ld)
    cp = params.c()
    if selection is None:
        selection = Selection(B, Hkv, params.k_blocks, cp.sample_cap, q.device,
                              draw_rows=Hq if params.per_head else None)
    ws = workspace(shape, cp, OP_SELECT, q.device)
    st = stats.c()
    sel = selection.c()
    _check(_lib().sa_select(ctypes.byref(shape), ctypes.byref(cp), _ptr(q), ctypes.byref(st), _ptr(k), _ptr(v),
                            ctypes.byref(sel), float(scale), _ptr(ws), ws.numel(), _stream(stream)),
           "sa_select")
    return selection


def decode(q, k, v, stats, selection, params, mode="resa", lam=1.0, scale=0.0, out=None, length=None,
           stream=None):
    B, Hq, d = q.shape
    shape = make_shape(k, Hq, length)
    cp = params.c()
    dp = sa_decode_params(MODES[mode], float(lam), float(scale))
    if out is None:
        out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
    ws = workspace(shape, cp, OP_DECODE, q.device)
    st = stats.c() if stats is not None else sa_stats()
    sel = selection.c()
    _check(_lib().sa_decode(ctypes.byref(shape), ctypes.byref(dp), ctypes.byref(cp), _ptr(q), _ptr(k), _ptr(v),
                            ctypes.byref(st), ctypes.byref(sel), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
           "sa_decode")
    return out


def step(q, k, v, stats, params, mode="resa", lam=1.0, scale=0.0, selection=None, out=None, length=None,
         stream=None):
    """Selection then decode in one call: the two kernels with the decode
    overlapping the end of the selection (programmatic dependent launch).
    Returns (out, selection)."""
    B, Hq, d = q.shape
    shape = make_shape(k, Hq, length)
    cp = params.c()
    dp = sa_decode_params(MODES[mode], float(lam), float(scale))
    if selection is None:
        selection = Selection(B, shape.Hkv, params.k_blocks, cp.sample_cap, q.device,
                              draw_rows=Hq if params.per_head else None)
    if out is None:
        out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
    ws = workspace(shape, cp, OP_STEP, q.device)
    st = stats.c()
    sel = selection.c()
    _check(_lib().sa_step(ctypes.byref(shape), ctypes.byref(dp), ctypes.byref(cp), _ptr(q), _ptr(k), _ptr(v),
                          ctypes.byref(st), ctypes.byref(sel), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
           "sa_step")
    return out, selection


class PreparedStep:
    """The arguments of sa_step built once for a fixed cache, statistics,
    parameters and selection buffers; each call passes this step's query and
    output (and optionally the decode step index that keys the draws) and
    runs one sa_step.  For callers that decode many steps with the same
    buffers: a call marshals two pointers and the stream instead of
    rebuilding every structure."""

    def __init__(self, k, v, stats, params, mode="resa", lam=1.0, scale=0.0, selection=None, length=None,
                 Hq=None):
        B, Hkv, ld, d = k.shape
        Hq = stats.mu_q.shape[1] if Hq is None else Hq
        self.k, self.v, self.stats = k, v, stats
        self.shape = make_shape(k, Hq, length)
        self.cp = params.c()
        self.dp = sa_decode_params(MODES[mode], float(lam), float(scale))
        self.selection = selection if selection is not None else Selection(
            B, Hkv, params.k_blocks, self.cp.sample_cap, k.device, draw_rows=Hq if params.per_head else None)
        self.ws = workspace(self.shape, self.cp, OP_STEP, k.device)
        self._st = stats.c()
        self._sel = self.selection.c()
        self._args = (ctypes.byref(self.shape), ctypes.byref(self.dp), ctypes.byref(self.cp))
        self._tail = (_ptr(k), _ptr(v), ctypes.byref(self._st), ctypes.byref(self._sel))
        self._ws = (_ptr(self.ws), self.ws.numel())
        self._fn = _lib().sa_step

    def __call__(self, q, out, step=None, stream=None):
        if step is not None:
            self.cp.step = int(step)
        _check(self._fn(*self._args, ctypes.c_void_p(q.data_ptr()), *self._tail, ctypes.c_void_p(out.data_ptr()),
                        *self._ws, _stream(stream)), "sa_step")
        return out


def dense_decode(q, k, v, scale=0.0, out=None, length=None, stream=None):
    B, Hq, d = q.shape
    shape = make_shape(k, Hq, length)
    if out is None:
        out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
    ws = workspace(shape, None, OP_DENSE, q.device)
    _check(_lib().sa_dense_decode(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(out), float(scale),
                                  _ptr(ws), ws.numel(), _stream(stream)), "sa_dense_decode")
    return out


def append(k_new, v_new, k, v, stats, length, scale=0.0, stream=None):
    """Writes one token per unit (k_new, v_new [B, Hkv, d]) at position
    `length` of the cache k, v [B, Hkv, ld, d] and refreshes the statistics
    (see sa_append).  Returns the new length."""
    shape = make_shape(k, stats.mu_q.shape[1], length)
    st = stats.c()
    _check(_lib().sa_append(ctypes.byref(shape), _ptr(k_new), _ptr(v_new), _ptr(k), _ptr(v), ctypes.byref(st),
                            float(scale), _stream(stream)), "sa_append")
    return int(length) + 1


def wait_timeouts():
    """Selection CTAs on the current device that gave up waiting on a bulk copy
    since the library was loaded (cumulative; see sa_wait_timeouts)."""
    c = ctypes.c_uint(0)
    _check(_lib().sa_wait_timeouts(ctypes.byref(c)), "sa_wait_timeouts")
    return int(c.value)
