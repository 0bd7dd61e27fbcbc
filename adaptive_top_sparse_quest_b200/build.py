"""Build the sm_100a C-ABI library libtwilight.so in-tree with nvcc.

    python -m adaptive_top_sparse_quest_b200.build [--force]
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_DIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIB_DIR, "libtwilight.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    for c in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found: cannot build the Twilight CUDA library")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")) +
                              glob.glob(os.path.join(CSRC, "*.h")) +
                              glob.glob(os.path.join(INCLUDE, "*.h")))


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _deps())


def _objdir() -> str:
    return os.path.join(LIB_DIR, "obj")


def build(force: bool = False, verbose: bool = False, extra_flags=None) -> str:
    """Compile every .cu under csrc/ (one nvcc process per file, in parallel)
    and link lib/libtwilight.so (sm_100a)."""
    if not force and up_to_date():
        return LIB
    import concurrent.futures as cf
    os.makedirs(_objdir(), exist_ok=True)
    nvcc = _nvcc()
    compile_flags = [f for f in NVCC_FLAGS if f != "-shared"]
    srcs = sources()

    def one(src):
        obj = os.path.join(_objdir(), os.path.basename(src)[:-3] + ".o")
        cmd = [nvcc, *compile_flags, *(extra_flags or []), "-I", INCLUDE, "-I", CSRC, "-c",
               "-o", obj, src]
        r = subprocess.run(cmd, capture_output=True, text=True)
        return src, obj, cmd, r

    keep = {os.path.basename(x)[:-3] + ".o" for x in srcs}
    for f in os.listdir(_objdir()):   # objects of sources that no longer exist
        if f.endswith(".o") and f not in keep:
            os.remove(os.path.join(_objdir(), f))
    objs = []
    with cf.ThreadPoolExecutor(max_workers=max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
        for src, obj, cmd, r in ex.map(one, srcs):
            if verbose:
                print(" ".join(cmd), flush=True)
            if r.returncode != 0:
                raise RuntimeError(f"nvcc failed on {src}:\n" + r.stdout + r.stderr)
            if verbose and (r.stdout or r.stderr):
                print(r.stdout + r.stderr)
            objs.append(obj)
    tmp = LIB + ".tmp"
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-Xcompiler", "-fPIC",
           "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc link failed:\n" + r.stdout + r.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None)
    print(LIB)
