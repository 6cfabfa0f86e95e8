"""Builds the CUDA library libgradsolve_b200.so in-tree for sm_100a with nvcc, and its checked
variant libgradsolve_b200_checked.so (-DGS_CHECKED: accesses through a record's chunk table are
bounds-checked, counted and redirected; see gs_checked_violations).

    python -m differentiable_adaptive_ode_b200.build [--force] [--checked] [-v]
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libgradsolve_b200.so")
CHECKED_LIB = os.path.join(PKG, "libgradsolve_b200_checked.so")
SOURCES = ["gs_api.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _deps():
    out = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh"))]
    out.append(os.path.join(INCLUDE, "gradsolve_b200.h"))
    return out


def nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    lib = CHECKED_LIB if checked else LIB
    if not force and os.path.exists(lib):
        if os.path.getmtime(lib) >= max(os.path.getmtime(p) for p in _deps()):
            return lib
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [nvcc(), "-std=c++20", "-O3", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
           "-I" + INCLUDE, "-o", tmp] + [os.path.join(CSRC, s) for s in SOURCES]
    if checked:
        cmd.insert(1, "-DGS_CHECKED")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                checked="--checked" in sys.argv))
