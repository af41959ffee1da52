"""Builds libtp.so (CUDA C++ for sm_100a) in-tree.

Steps: run csrc/codegen.py (tables and unrolled bodies into csrc/gen/), compile every
translation unit with nvcc in parallel, link one shared library next to this file.
Incremental: a unit is recompiled only when a source or header is newer than its object.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
GEN = os.path.join(CSRC, "gen")
OBJ = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libtp.so")
ROOT = os.path.dirname(HERE)

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--use_fast_math",
              "-Xptxas", "-O3", "-I", CSRC, "-I", GEN, "-I", os.path.join(ROOT, "include")]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu"))) + sorted(glob.glob(os.path.join(GEN, "*.cu")))
    headers = (glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))
               + glob.glob(os.path.join(GEN, "*.h")) + glob.glob(os.path.join(ROOT, "include", "*.h")))
    return srcs, headers


def _compile(nvcc, src, obj, verbose_ptxas=False):
    cmd = [nvcc, *ARCH, *NVCC_FLAGS, "-c", src, "-o", obj]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    t = time.time()
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stderr[-6000:]}")
    return os.path.basename(src), time.time() - t, r.stderr


def build(jobs: int | None = None, verbose: bool = False, ptxas_v: bool = False) -> str:
    sys.path.insert(0, CSRC)
    try:
        import codegen  # noqa: E402
    finally:
        sys.path.pop(0)
    codegen.main(GEN)
    os.makedirs(OBJ, exist_ok=True)
    nvcc = _nvcc()
    srcs, headers = _sources()
    hdr_mtime = max(os.path.getmtime(h) for h in headers)
    todo = []
    objs = []
    for s in srcs:
        o = os.path.join(OBJ, os.path.splitext(os.path.basename(s))[0] + ".o")
        objs.append(o)
        if (not os.path.exists(o) or os.path.getmtime(o) < max(os.path.getmtime(s), hdr_mtime)
                or ptxas_v):
            todo.append((s, o))
    jobs = jobs or max(1, len(os.sched_getaffinity(0)))
    logs = []
    with cf.ThreadPoolExecutor(jobs) as ex:
        for name, dt, err in ex.map(lambda so: _compile(nvcc, so[0], so[1], ptxas_v), todo):
            logs.append((name, dt, err))
            if verbose:
                print(f"  compiled {name} in {dt:.1f}s", flush=True)
    if todo or not os.path.exists(LIB):
        cmd = [nvcc, *ARCH, "-shared", "-o", LIB + ".tmp", *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n" + r.stderr[-4000:])
        os.replace(LIB + ".tmp", LIB)
    if ptxas_v:
        for name, _, err in logs:
            print(f"== {name}\n{err}")
    return LIB


if __name__ == "__main__":
    t0 = time.time()
    path = build(verbose=True, ptxas_v="-v" in sys.argv)
    print(f"built {path} in {time.time() - t0:.1f}s")
