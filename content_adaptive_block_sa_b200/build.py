"""Builds libsa.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m content_adaptive_block_sa_b200.build [--force]

Objects go to ``content_adaptive_block_sa_b200/_build/`` and the shared
library to ``content_adaptive_block_sa_b200/libsa.so``; the instrumented
variant with tile counters (``-DSA_COUNT_TILES``) to ``_build_count/`` and
``libsa_count.so``. A source is
recompiled when it, or any header, is newer than its object.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libsa.so")
# instrumented variant: the same library with per-call tile counters in the
# status header (-DSA_COUNT_TILES), loaded only by the tests that check them
BUILD_COUNT = os.path.join(PKG, "_build_count")
LIB_COUNT = os.path.join(PKG, "libsa_count.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I", INCLUDE, "-I", CSRC]


def _newest(paths):
    return max((os.path.getmtime(p) for p in paths), default=0.0)


def _run(cmd):
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("command failed: " + " ".join(cmd) + "\n" + r.stdout + r.stderr)
    return r.stdout + r.stderr


def build(force: bool = False, verbose: bool = False, extra_flags=None, count_tiles=False) -> str:
    """Builds libsa.so (or, with count_tiles, the instrumented libsa_count.so)."""
    build_dir, lib = (BUILD_COUNT, LIB_COUNT) if count_tiles else (BUILD, LIB)
    os.makedirs(build_dir, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = (glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
               + glob.glob(os.path.join(INCLUDE, "*.h")))
    h_time = _newest(headers)
    extra = list(extra_flags or []) + (["-DSA_COUNT_TILES"] if count_tiles else [])

    def compile_one(src):
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        if force or not os.path.exists(obj) or os.path.getmtime(obj) < max(os.path.getmtime(src), h_time):
            out = _run([NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj])
            if verbose and out.strip():
                print(out)
        return obj

    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, sources))
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < _newest(objs):
        _run([NVCC, *ARCH, "-shared", "-o", lib, *objs, "-lcudart"])
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, count_tiles=True))
