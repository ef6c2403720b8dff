"""Build the package's shared libraries in-tree with nvcc for sm_100a:
libalspec.so (the decode library, include/alspec.h), libalspec_debug.so
(the same library with the kernels' bounds checks compiled in,
ALSPEC_DEBUG_BOUNDS: an index outside its buffer sets ALSPEC_DEVERR_BOUNDS
in the device error word and the access is skipped) and
libalspec_read_probe.so (the benchmark's read-bandwidth probe,
include/alspec_read_probe.h).

Usage: python speculative_flash_decoding_b200/build.py [--force] [-v]
(run by path: importing the package needs the built library)
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libalspec.so")
DEBUG_LIB = os.path.join(PKG, "libalspec_debug.so")
PROBE_LIB = os.path.join(PKG, "libalspec_read_probe.so")
_DECODE_DEPS = ([os.path.join(CSRC, f) for f in ("attn_kernels.cuh", "oproj_kernels.cuh",
                                                 "ptx.cuh")] +
                [os.path.join(INCLUDE, "alspec.h")])
# (library, its source, the headers it depends on, extra nvcc flags)
TARGETS = [
    (LIB, os.path.join(CSRC, "alspec.cu"), _DECODE_DEPS, []),
    (DEBUG_LIB, os.path.join(CSRC, "alspec.cu"), _DECODE_DEPS, ["-DALSPEC_DEBUG_BOUNDS"]),
    (PROBE_LIB, os.path.join(CSRC, "read_probe.cu"),
     [os.path.join(CSRC, "ptx.cuh"), os.path.join(INCLUDE, "alspec_read_probe.h")], []),
]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC", "-cudart", "static",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _build_one(lib: str, src: str, deps, flags, force: bool, verbose: bool) -> None:
    if not force and os.path.exists(lib):
        newest = max(os.path.getmtime(p) for p in [src, *deps])
        if os.path.getmtime(lib) >= newest:
            return
    tmp = lib + ".tmp"
    cmd = [nvcc(), *NVCC_FLAGS, *flags, "-I", INCLUDE, "-I", CSRC, "-o", tmp, src]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every library of the package; return the decode library's path."""
    for lib, src, deps, flags in TARGETS:
        _build_one(lib, src, deps, flags, force, verbose)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
