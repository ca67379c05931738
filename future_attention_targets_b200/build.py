"""Builds the C-ABI library libkvpop.so in-tree with nvcc for sm_100a."""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libkvpop.so")
DEBUG_LIB = os.path.join(PKG, "libkvpop_debug.so")   # the same sources with KVPOP_DEBUG bounds checks

NVCC_FLAGS = [
    "-std=c++17", "-O3", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; the CUDA toolkit is needed to build libkvpop.so")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) \
        + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra_flags: list[str] | None = None,
          debug: bool = False) -> str:
    """Compiles every CUDA source into libkvpop.so, or with debug=True into libkvpop_debug.so (the same
    sources with every kernel's bounds checks compiled in, KVPOP_DEBUG); skipped when up to date."""
    lib = DEBUG_LIB if debug else LIB
    if not force and not _stale(lib):
        return lib
    tmp = lib + ".tmp"
    flags = [*NVCC_FLAGS, *(["-DKVPOP_DEBUG"] if debug else []), *(extra_flags or [])]
    cmd = [_nvcc(), *flags, "-I", INCLUDE, "-I", CSRC, "-shared",
           *sources(), "-o", tmp, "-lcudart_static", "-ldl", "-lrt", "-lpthread"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    force = "--force" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []
    print(build(force=force or bool(extra), verbose=True, extra_flags=extra, debug="--debug" in sys.argv))
