"""Builds libwkv4.so in-tree: nvcc for sm_100a, CUDA runtime linked statically.

    python -m rwkv_wkv_linear_b200._build [--force]
"""

from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libwkv4.so")
# the bounds-checked build (WKV4_CHECKED: every global index checked, fault
# injection switches read from the environment), for the failure tests
CHECKED_LIB = os.path.join(PKG, "libwkv4_checked.so")
SOURCES = [os.path.join(CSRC, "wkv4_kernels.cu"), os.path.join(CSRC, "wkv4_api.cpp"),
           os.path.join(CSRC, "wkv4_host.cpp")]


def deps():
    """Every source the library is built from: all of csrc/ and include/."""
    out = []
    for d in (CSRC, INCLUDE):
        out += [os.path.join(d, f) for f in sorted(os.listdir(d))
                if f.endswith((".cu", ".cuh", ".cpp", ".h"))]
    return out

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared", "-cudart", "static",
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(d) > t for d in deps())


def stale_at(path: str) -> bool:
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    return any(os.path.getmtime(d) > t for d in deps())


def build_checked(force: bool = False, verbose: bool = False) -> str:
    """Compile libwkv4_checked.so (WKV4_CHECKED) when stale."""
    if not force and not stale_at(CHECKED_LIB):
        return CHECKED_LIB
    return build(force=True, verbose=verbose, out=CHECKED_LIB, defines=("WKV4_CHECKED",))


def build(force: bool = False, verbose: bool = False, out: str = LIB, defines=()) -> str:
    """Compile libwkv4.so (or `out`, with extra -D `defines`) when stale."""
    if out == LIB and not defines and not force and not stale():
        return LIB
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *[f"-D{d}" for d in defines], "-I", INCLUDE, "-o", tmp, *SOURCES]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
    print(build_checked(force="--force" in sys.argv, verbose=True))
