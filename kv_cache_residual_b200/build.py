"""Build libsa_b200.so in-tree with nvcc for sm_100a.

    python -m kv_cache_residual_b200.build          # incremental
    python -m kv_cache_residual_b200.build --force  # rebuild everything

Each CUDA source compiles to an object under _build/ (git-ignored), then
one shared library is linked next to this file.  Also compiles the optional
C part of the oracle when present (none today).
"""
import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libsa_b200.so")
SOURCES = ["sa_api.cu", "sa_prefill.cu", "sa_select.cu", "sa_decode.cu", "sa_clt.cu", "sa_select_var.cu", "sa_multi.cu", "sa_qgc.cu", "sa_noalloc.cu",
           "sa_append.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "-I", os.path.join(ROOT, "include")]


def nvcc():
    for c in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _deps_mtime():
    m = 0.0
    for d in (CSRC, os.path.join(ROOT, "include")):
        for f in os.listdir(d):
            if f.endswith((".cuh", ".h")):
                m = max(m, os.path.getmtime(os.path.join(d, f)))
    return m


def _compile(src, obj, verbose):
    cmd = [nvcc()] + ARCH + FLAGS + (["-Xptxas", "-v"] if verbose else []) + ["-c", os.path.join(CSRC, src), "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed for %s:\n%s\n%s" % (src, " ".join(cmd), r.stderr))
    return r.stderr


def build(force=False, verbose=False):
    os.makedirs(BUILD, exist_ok=True)
    dep = _deps_mtime()
    todo = []
    objs = []
    for s in SOURCES:
        o = os.path.join(BUILD, s.replace(".cu", ".o"))
        objs.append(o)
        if force or not os.path.exists(o) or os.path.getmtime(o) < max(dep, os.path.getmtime(os.path.join(CSRC, s))):
            todo.append((s, o))
    logs = {}
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        futs = {ex.submit(_compile, s, o, verbose): s for s, o in todo}
        for f in cf.as_completed(futs):
            logs[futs[f]] = f.result()
    if todo or force or not os.path.exists(LIB):
        cmd = [nvcc()] + ARCH + ["-shared", "-o", LIB] + objs + ["-lcudart"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n%s" % r.stderr)
    return LIB, logs


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true", help="print register / shared-memory usage")
    a = ap.parse_args()
    lib, logs = build(force=a.force or a.ptxas_v, verbose=a.ptxas_v)
    for s, log in sorted(logs.items()):
        if a.ptxas_v and log:
            print("==", s)
            print(log)
    print(lib)


if __name__ == "__main__":
    sys.exit(main())
