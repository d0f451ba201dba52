"""Builds libsolattn.so (the C-ABI library) in place with nvcc for sm_100a.

Usage: python -m video_diffusion_b200.build [--force] [--ptxas-info] [--debug]
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libsolattn.so")
DEBUG_LIB = os.path.join(HERE, "libsolattn_debug.so")  # consistency checks on (tests only)
SOURCES = ["api.cu", "prologue.cu", "attn_tc.cu", "attn_simt.cu"]
HEADERS = ["common.cuh", "sm100.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libsolattn")


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "sol_attn.h"),
                                                                  os.path.abspath(__file__)]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, ptxas_info: bool = False, debug: bool = False) -> str:
    """Builds the release library, or (debug=True) the variant whose kernels
    record failed consistency checks in the device status word."""
    lib = DEBUG_LIB if debug else LIB
    if not force and not ptxas_info and not _stale(lib):
        return lib
    cmd = [nvcc_path(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
           "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE, "-o", lib + ".tmp"]
    if debug:
        cmd += ["-DSOL_ATTN_DEBUG_CHECKS"]
    if ptxas_info:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    proc = subprocess.run(cmd, capture_output=True, text=True)
    if proc.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + proc.stdout + proc.stderr)
    os.replace(lib + ".tmp", lib)
    if ptxas_info:
        sys.stderr.write(proc.stderr)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, ptxas_info="--ptxas-info" in sys.argv, debug="--debug" in sys.argv))
