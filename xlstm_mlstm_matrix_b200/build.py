"""Builds the C-ABI library ``libxlstm_mlstm.so`` in-tree with nvcc for sm_100a.

Run as ``python -m xlstm_mlstm_matrix_b200.build`` (or through
``__graft_entry__.build()``).  Objects are compiled in parallel and cached by
source/flags hash under ``_build/``; the shared library lands next to this file.
"""
from __future__ import annotations

import concurrent.futures as cf
import hashlib
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OUT = os.path.join(HERE, "libxlstm_mlstm.so")
# tcgen05 issue-cost microbenchmark (measurement tooling, driven by bench.py --probe mma)
PROBE_SRC = os.path.join(CSRC, "probe", "mma_cost.cu")
PROBE_OUT = os.path.join(HERE, "libxlstm_mma_probe.so")
BUILD_DIR = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills", "-I" + INCLUDE, "-I" + CSRC]


def nvcc() -> str:
    cand = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA library cannot be built")
    return cand


def _sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _deps_hash(src: str, flags) -> str:
    h = hashlib.sha256()
    h.update(" ".join(flags).encode())
    h.update(open(src, "rb").read())
    for f in sorted(os.listdir(CSRC)):
        if f.endswith((".cuh", ".h")):
            h.update(open(os.path.join(CSRC, f), "rb").read())
    h.update(open(os.path.join(INCLUDE, "xlstm_mlstm.h"), "rb").read())
    return h.hexdigest()[:16]


def _compile(src: str, extra) -> str:
    flags = NVCC_FLAGS + ARCH + list(extra)
    obj = os.path.join(BUILD_DIR, os.path.basename(src) + "." + _deps_hash(src, flags) + ".o")
    if not os.path.exists(obj):
        tmp = obj + f".tmp{os.getpid()}"
        subprocess.check_call([nvcc(), "-c", src, "-o", tmp] + flags)
        os.replace(tmp, obj)
    return obj


def build(verbose: bool = False, extra=()) -> str:
    os.makedirs(BUILD_DIR, exist_ok=True)
    srcs = _sources()
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra), srcs))
    tmp = OUT + f".tmp{os.getpid()}"
    subprocess.check_call([nvcc(), "-shared", "-o", tmp] + objs + ARCH)
    os.replace(tmp, OUT)
    probe = _compile(PROBE_SRC, extra)
    tmp = PROBE_OUT + f".tmp{os.getpid()}"
    subprocess.check_call([nvcc(), "-shared", "-o", tmp, probe] + ARCH)
    os.replace(tmp, PROBE_OUT)
    if verbose:
        print(OUT)
    return OUT


if __name__ == "__main__":
    build(verbose=True, extra=sys.argv[1:])
