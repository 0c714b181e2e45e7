"""Builds liblora_linear.so in-tree with nvcc for sm_100a.

    python qlora_linear_b200/build.py        (or __graft_entry__.build())
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "liblora_linear.so")
# The checked build: every TMA producer tests its tile coordinates and box origins before
# a copy and reports LORA_ERR_DEVICE_BOUNDS instead of issuing an out-of-range one
# (select it with LORA_LIB_PATH; the tests run the ragged shapes on it).
LIB_CHECKED = os.path.join(PKG, "liblora_linear_checked.so")
SOURCES = ["lora_api.cu"]
HEADERS = ["ptx.cuh", "dequant.cuh", "gemm_common.cuh", "gemm_pair.cuh", "gemm_q.cuh", "skinny.cuh", "dualproj.cuh",
           "elementwise.cuh", "streamk.cuh", "tcproj.cuh"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def flags(extra=()) -> list[str]:
    return [
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-O3", "-lineinfo", "-std=c++17",
        "-Xcompiler", "-fPIC", "-shared",
        "--expt-relaxed-constexpr",
        "-I", INCLUDE, "-I", CSRC,
        *extra,
    ]


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra=(), checked: bool = False) -> str:
    """Compile the library (or its checked build) if any source is newer than it; returns
    the .so path."""
    lib = LIB_CHECKED if checked else LIB
    if checked:
        extra = (*extra, "-DLORA_CHECKED=1")
    if not force and not _stale(lib):
        return lib
    tmp = lib + ".tmp"
    cmd = [nvcc_path(), *flags(extra), "-o", tmp, *[os.path.join(CSRC, s) for s in SOURCES]]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose and (res.stdout or res.stderr):
        print(res.stdout + res.stderr)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=("-Xptxas", "-v") if "--ptxas-v" in sys.argv else (), checked="--checked" in sys.argv)
