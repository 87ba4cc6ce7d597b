"""Build the in-tree shared libraries.

* ``libtm.so``        - the CUDA library behind ``include/tm.h`` (sm_100a only).
* ``inputs/libtm_inputs.so`` - the seeded input generator (plain C).

Both are built in place so that they travel with the source tree; nvcc
cross-compiles sm_100a without a GPU.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBTM = os.path.join(PKG, "libtm.so")
LIBINPUTS = os.path.join(PKG, "inputs", "libtm_inputs.so")

NVCC_ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(target: str, sources) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def build_inputs(force: bool = False) -> str:
    src = os.path.join(PKG, "inputs", "tm_inputs.c")
    if force or _stale(LIBINPUTS, [src]):
        subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", src, "-lm",
                        "-o", LIBINPUTS], check=True)
    return LIBINPUTS


def cuda_sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def build_lib(force: bool = False, verbose_ptxas: bool = False, extra=()) -> str:
    srcs = cuda_sources()
    deps = srcs + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    if not srcs:
        raise RuntimeError("no CUDA sources")
    if not (force or _stale(LIBTM, deps)):
        return LIBTM
    cmd = [_nvcc(), *NVCC_ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "-I", INCLUDE, "-I", CSRC, *srcs, "-o", LIBTM]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    cmd[1:1] = list(extra)
    subprocess.run(cmd, check=True)
    return LIBTM


def build_all(force: bool = False) -> None:
    build_inputs(force)
    build_lib(force)


if __name__ == "__main__":
    import sys
    build_all(force="--force" in sys.argv)
