"""Builds libmoba.so (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: ``python -m block_sparse_long_meanpool_b200.build [--verbose]``.  The CUDA runtime is
linked statically, so the library loads (and exports its symbols) on a machine without a
GPU; it needs the NVIDIA driver only when a function is called.
"""

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libmoba.so")
SOURCES = ["moba_api.cu", "meanpool.cu", "gate.cu", "gate_tc.cu", "route.cu", "attn_tc.cu", "merge.cu", "decode.cu", "minmaxpool.cu", "noalloc.cu", "attn_bwd.cu"]
HEADERS = ["moba_internal.cuh", "ptx.cuh"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "-cudart", "static",
         "--expt-relaxed-constexpr"]


def nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "moba.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def _run(cmd):
    proc = subprocess.run(cmd, capture_output=True, text=True)
    if proc.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + proc.stdout + proc.stderr)
    return proc.stdout + proc.stderr


def build(force=False, verbose=False):
    """Compile every source into libmoba.so unless it is up to date.  Returns its path.

    Each source is compiled to its own object in parallel (build/ beside the sources), then
    the objects are linked into the shared library."""
    if not force and not _stale():
        return LIB
    objdir = os.path.join(PKG, "build")
    os.makedirs(objdir, exist_ok=True)
    base = [nvcc()] + ARCH + FLAGS + ["-I", os.path.join(ROOT, "include"), "-I", CSRC]
    if verbose:
        base += ["-Xptxas", "-v"]
    objs, cmds = [], []
    for f in SOURCES:
        obj = os.path.join(objdir, f.replace(".cu", ".o"))
        objs.append(obj)
        cmds.append(base + ["-c", "-o", obj, os.path.join(CSRC, f)])
    workers = max(1, min(len(cmds), os.cpu_count() or 1))
    with ThreadPoolExecutor(workers) as pool:
        logs = list(pool.map(_run, cmds))
    if verbose:
        sys.stderr.write("".join(logs))
    _run([nvcc()] + ARCH + ["-cudart", "static", "-shared", "-o", LIB + ".tmp"] + objs)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
