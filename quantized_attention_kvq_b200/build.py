"""Build the package's native libraries in-tree.

* ``lib/libkvq.so``    -- the C-ABI library (CUDA, sm_100a only), from ``csrc/*.cu``.
* ``lib/libkvq_checked.so`` -- the same with -DKVQ_BOUNDS_CHECK: every checked
  cache, partial and window access compares its range with the array's extent,
  skips and counts an access out of bounds (``kvq_bounds_violations``).
* ``lib/libkvqgen.so`` -- the seeded input generator (plain C + OpenMP).

The quantizer inside libkvq relies on IEEE-rounded fp32 subtract/divide and
fp64 adds, so nothing here passes fast-math flags.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB_DIR = os.path.join(PKG, "lib")
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(ROOT, "_build")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _newer(target: str, sources: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def build_gen(force: bool = False) -> str:
    os.makedirs(LIB_DIR, exist_ok=True)
    src = os.path.join(PKG, "synth", "kvqgen.c")
    so = os.path.join(LIB_DIR, "libkvqgen.so")
    if force or _newer(so, [src]):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", so, src, "-lm"])
    return so


def build_kvq(force: bool = False, verbose_ptxas: bool = False, checked: bool = False) -> str:
    os.makedirs(LIB_DIR, exist_ok=True)
    build_dir = BUILD_DIR + ("_checked" if checked else "")
    os.makedirs(build_dir, exist_ok=True)
    so = os.path.join(LIB_DIR, "libkvq_checked.so" if checked else "libkvq.so")
    extra = ["-DKVQ_BOUNDS_CHECK"] if checked else []
    cus = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdrs = sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h")))
    objs = []
    jobs = []
    for cu in cus:
        obj = os.path.join(build_dir, os.path.basename(cu) + ".o")
        objs.append(obj)
        if force or _newer(obj, [cu] + hdrs):
            cmd = [NVCC, *ARCH, *NVCC_FLAGS, *extra, "-c", cu, "-o", obj]
            if verbose_ptxas:
                cmd[1:1] = ["-Xptxas", "-v"]
            jobs.append(cmd)
    if jobs:
        with ThreadPoolExecutor(max_workers=min(8, len(jobs))) as ex:
            for rc, cmd in zip(ex.map(lambda c: subprocess.call(c), jobs), jobs):
                if rc != 0:
                    raise RuntimeError("nvcc failed: " + " ".join(cmd))
    if force or jobs or _newer(so, objs):
        subprocess.check_call([NVCC, *ARCH, "-shared", "-o", so, *objs, "-lcudart"])
    return so


def build_all(force: bool = False) -> None:
    build_gen(force)
    build_kvq(force)
    build_kvq(force, checked=True)


if __name__ == "__main__":
    build_all(force="--force" in sys.argv)
    print("built", LIB_DIR)
