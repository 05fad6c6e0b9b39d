"""Compile the CUDA library (sm_100a) in-tree: libmamba_mixer.so next to this
file, and its checked build libmamba_mixer_checked.so (compiled with
MM_CHECK_BOUNDS: the forward and decode kernels check every index they form
against its buffer, skip an access outside it and report MM_ERR_BOUNDS).

    python -m mamba_selective_scan_core_b200.build [--force] [--verbose] [--checked]
"""

from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
INCLUDE = os.path.join(ROOT, "include")
CSRC = os.path.join(PKG, "csrc")
SOURCE = os.path.join(CSRC, "mixer_api.cu")
LIB_PATH = os.path.join(PKG, "libmamba_mixer.so")
CHECKED_LIB_PATH = os.path.join(PKG, "libmamba_mixer_checked.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC",
]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build the mixer library")


def _inputs():
    return [SOURCE] + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def stale(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    return any(os.path.getmtime(f) > t for f in _inputs())


def _compile(path: str, flags, verbose: bool) -> str:
    tmp = path + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *NVCC_FLAGS, *flags, "-I", INCLUDE, "-o", tmp, SOURCE]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, path)
    return path


def build(force: bool = False, verbose: bool = False, extra_flags=()) -> str:
    if not force and not stale(LIB_PATH):
        return LIB_PATH
    return _compile(LIB_PATH, list(extra_flags), verbose)


def build_checked(force: bool = False, verbose: bool = False) -> str:
    """The checked build (index checks in the forward and decode kernels)."""
    if not force and not stale(CHECKED_LIB_PATH):
        return CHECKED_LIB_PATH
    return _compile(CHECKED_LIB_PATH, ["-DMM_CHECK_BOUNDS"], verbose)


if __name__ == "__main__":
    if "--checked" in sys.argv:
        print(build_checked(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
    else:
        print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
