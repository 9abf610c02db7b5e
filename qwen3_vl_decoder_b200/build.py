"""Builds libq3vl.so in-tree from csrc/ for sm_100a with nvcc.

    python -m qwen3_vl_decoder_b200.build [--force] [--debug]

Objects go to ``_build/`` at the repository root; the shared library is
written next to this file. ``--debug`` builds ``libq3vl_debug.so`` instead
(objects in ``_build/debug``), compiled with ``-DQ3VL_DEBUG``: the kernels
then check the computed index of every global access they make outside TMA
and record Q3VL_ERANGE instead of making an out-of-range access. Load it
with ``Q3VL_LIBRARY=debug`` in the environment. The CUDA runtime is linked statically and the
driver API is reached through the runtime's entry-point query, so the
library loads on a machine without a GPU driver (its calls then fail with
an error status).
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libq3vl.so")
LIB_DEBUG = os.path.join(PKG, "libq3vl_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I" + INCLUDE, "-I" + CSRC]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _deps():
    return [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "q3vl.h")]


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compiles every source that changed and links the library; returns its path."""
    bdir = os.path.join(BUILD, "debug") if debug else BUILD
    lib = LIB_DEBUG if debug else LIB
    flags = FLAGS + (["-DQ3VL_DEBUG"] if debug else [])
    os.makedirs(bdir, exist_ok=True)
    nvcc = _nvcc()
    deps = _deps()
    jobs = []
    for src in _sources():
        obj = os.path.join(bdir, os.path.basename(src)[:-3] + ".o")
        if force or _stale(obj, deps):
            jobs.append([nvcc, *ARCH, *flags, "-c", src, "-o", obj])
    objs = [os.path.join(bdir, os.path.basename(s)[:-3] + ".o") for s in _sources()]

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
        if verbose and (r.stdout or r.stderr):
            print(r.stdout + r.stderr, file=sys.stderr)

    with cf.ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        list(ex.map(run, jobs))
    if force or jobs or _stale(lib, objs):
        run([nvcc, *ARCH, "-shared", "-cudart", "static", "-o", lib, *objs])
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                debug="--debug" in sys.argv))
