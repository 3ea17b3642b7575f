"""Build libeqw.so in-tree with nvcc for sm_100a (B200).

Usage: ``python -m entropy_coded_weight_b200.build [--force] [--verbose]``.
Compiles every source under ``csrc/`` (CUDA with -O3 -lineinfo, no fast-math,
denormals kept, no FMA contraction in the dequantiser's explicit __fmul_rn;
host C++ with -O3) and links one shared library next to this file.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libeqw.so")
LIB_CHECKED = os.path.join(HERE, "libeqw_checked.so")  # EQ_CHECKED=1: run-time checks of the kernels' invariants
GENCODE = "-gencode=arch=compute_100a,code=sm_100a"


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: cannot build libeqw.so")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, defines: dict | None = None, out: str | None = None,
          checked: bool = False) -> str:
    """Compile and link libeqw.so.  ``defines`` (-D NAME=VALUE for the CUDA
    sources, e.g. EQ_SHARED_WARPS) and ``out`` build a tuning variant
    elsewhere; ``checked`` builds libeqw_checked.so (EQ_CHECKED=1), whose
    kernels test their invariants at run time (EQ_DEV_CHECK)."""
    if checked:
        defines = dict(defines or {}, EQ_CHECKED=1)
        if out is None and not force and not _stale(LIB_CHECKED):
            return LIB_CHECKED
        out = out or LIB_CHECKED
    target = out or LIB
    if not force and out is None and not _stale():
        return LIB
    nvcc = _nvcc()
    objdir = os.path.join(os.path.dirname(target), "_build", os.path.basename(target)) if out else \
        os.path.join(HERE, "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        if src.endswith(".cu"):
            cmd = [nvcc, GENCODE, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden",
                   "-ftz=false", "-prec-div=true", "-prec-sqrt=true", "-I", INCLUDE, "-c", src, "-o", obj]
            cmd += [f"-D{k}={v}" for k, v in (defines or {}).items()]
            if verbose:
                cmd[1:1] = ["-Xptxas", "-v"]
        else:
            cuda_inc = os.path.join(os.path.dirname(os.path.dirname(os.path.realpath(nvcc))), "include")
            cmd = [os.environ.get("CXX", "g++"), "-O3", "-std=c++17", "-fPIC", "-fvisibility=hidden", "-pthread",
                   "-Wall", "-Wextra", "-I", INCLUDE, "-I", cuda_inc, "-c", src, "-o", obj]
            cmd += [f"-D{k}={v}" for k, v in (defines or {}).items()]
        subprocess.check_call(cmd)
        objs.append(obj)
    tmp = target + f".{os.getpid()}.tmp"
    subprocess.check_call([nvcc, GENCODE, "-shared", "-Xcompiler", "-pthread", "-o", tmp] + objs)
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--checked", action="store_true", help="build libeqw_checked.so (EQ_CHECKED=1)")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, checked=a.checked))
    sys.exit(0)
