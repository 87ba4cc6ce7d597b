"""Build the in-tree shared libraries.

* ``libtm.so``        - the CUDA library behind ``include/tm.h`` (sm_100a only).
* ``inputs/libtm_inputs.so`` - the seeded input generator (plain C).

Both are built in place so that they travel with the source tree; nvcc
cross-compiles sm_100a without a GPU.
"""
from __future__ import annotations

import glob
import hashlib
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


def _stamp(sources, cmd) -> str:
    """Digest of the build command and of every source file's path and bytes."""
    h = hashlib.sha256()
    h.update("\0".join(cmd).encode())
    for s in sorted(sources):
        h.update(os.path.relpath(s, ROOT).encode())
        with open(s, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _stale(target: str, sources, cmd) -> bool:
    """A library is rebuilt unless its stamp file holds the digest of the
    sources and command it would be built from now. File times are not used:
    a copied tree can leave a library that is older than its sources looking
    newer (or the reverse)."""
    if not os.path.exists(target) or not os.path.exists(target + ".stamp"):
        return True
    with open(target + ".stamp") as f:
        return f.read().strip() != _stamp(sources, cmd)


def _write_stamp(target: str, sources, cmd) -> None:
    with open(target + ".stamp", "w") as f:
        f.write(_stamp(sources, cmd) + "\n")


def build_inputs(force: bool = False) -> str:
    src = os.path.join(PKG, "inputs", "tm_inputs.c")
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", src, "-lm", "-o", LIBINPUTS]
    key = [c if c not in (src, LIBINPUTS) else os.path.relpath(c, ROOT) for c in cmd]
    if force or _stale(LIBINPUTS, [src], key):
        subprocess.run(cmd, check=True)
        _write_stamp(LIBINPUTS, [src], key)
    return LIBINPUTS


def cuda_sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def lib_inputs(extra=()):
    """(CUDA sources, every file the library depends on, nvcc flags)."""
    srcs = cuda_sources()
    deps = srcs + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    flags = [*extra, *NVCC_ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared",
             "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden"]
    return srcs, deps, flags


def build_lib(force: bool = False, verbose_ptxas: bool = False, extra=()) -> str:
    srcs, deps, flags = lib_inputs(extra)
    if not srcs:
        raise RuntimeError("no CUDA sources")
    if not (force or verbose_ptxas or _stale(LIBTM, deps, flags)):
        return LIBTM
    cmd = [_nvcc(), *flags, "-I", INCLUDE, "-I", CSRC, *srcs, "-o", LIBTM]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    if os.path.exists(LIBTM + ".stamp"):
        os.remove(LIBTM + ".stamp")  # no stamp while the library is being replaced
    subprocess.run(cmd, check=True)
    _write_stamp(LIBTM, deps, flags)
    return LIBTM


def build_all(force: bool = False) -> None:
    build_inputs(force)
    build_lib(force)


if __name__ == "__main__":
    import sys
    build_all(force="--force" in sys.argv)
