"""Build the in-tree shared library ``libmoedecode.so`` (sm_100a) with nvcc.

Usage: ``python -m mixture_experts_decode_gemv_b200.build [--force] [--ptxas-verbose]``.
The library is rebuilt only when a source or header is newer than it (or with ``--force``).
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmoedecode.so")

SOURCES = ["api.cu", "host_formats.cpp", "no_alloc.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libmoedecode.so")


def _inputs():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)
             if f.endswith((".cu", ".cuh", ".cpp", ".h"))]
    files += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    return files + [os.path.abspath(__file__)]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, ptxas_verbose: bool = False, quiet: bool = False,
          defines=(), out: str = None) -> str:
    """Compile the library; ``defines`` (e.g. ``("MOE_PHASE_TIMERS",)``) and ``out`` give a
    separately named variant build."""
    target = out or LIB
    if not force and not defines and out is None and up_to_date():
        return LIB
    cmd = [_nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
           "-cudart", "static", "--expt-relaxed-constexpr", "-I", INCLUDE,
           *[f"-D{d}" for d in defines],
           "-o", target + ".tmp", *[os.path.join(CSRC, s) for s in SOURCES]]
    if ptxas_verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    if not quiet:
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, cwd=CSRC, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if ptxas_verbose or (res.stderr.strip() and not quiet):
        print(res.stderr, file=sys.stderr)
    os.replace(target + ".tmp", target)
    return target


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    ap.add_argument("--define", action="append", default=[])
    ap.add_argument("--out", default=None)
    a = ap.parse_args()
    print(build(force=a.force, ptxas_verbose=a.ptxas_verbose, defines=a.define, out=a.out))
