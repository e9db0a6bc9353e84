"""Build ``libmoe.so`` (the CUDA library behind include/moe.h) in-tree.

One nvcc invocation compiles every kernel for sm_100a only
(``-gencode arch=compute_100a,code=sm_100a``) into a shared library next to
this file, with the CUDA runtime linked statically so the library loads on a
machine without a GPU driver (for the export checks) and needs nothing from
torch. ``--checks`` builds the index-checking variant ``libmoe_checks.so``
(``-DMOE_CHECKS``: every data-dependent row or expert index is checked before
use, and a bad one is recorded in the device error word and skipped).
Usage: ``python -m sparse_mixture_experts_route_b200.build [--checks] [--verbose]``.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libmoe.so")
LIB_CHECKS = os.path.join(HERE, "libmoe_checks.so")
SOURCES = [os.path.join(CSRC, "moe_api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + \
    [os.path.join(INCLUDE, "moe.h")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def flags(verbose: bool = False, checks: bool = False):
    f = ["-DMOE_CHECKS"] if checks else []
    f += ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
         "-Xcompiler", "-fPIC", "-shared", "-cudart", "static", "-I", INCLUDE, "-I", CSRC,
         "--expt-relaxed-constexpr"]
    if verbose:
        f += ["-Xptxas", "-v"]
    return f


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in DEPS)


def build(force: bool = False, verbose: bool = False, checks: bool = False) -> str:
    lib = LIB_CHECKS if checks else LIB
    if not force and up_to_date(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *flags(verbose, checks), *SOURCES, "-o", tmp]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, checks="--checks" in sys.argv))
