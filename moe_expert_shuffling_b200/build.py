"""Compile libmoeshuffle.so (the CUDA kernels and the C ABI) in-tree for sm_100a."""

from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmoeshuffle.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared", "-cudart", "static",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          out: str | None = None) -> str:
    """Compile the library (to `out`, default the package's libmoeshuffle.so) if a source is
    newer than it, or always with force.  Processes that start together (one per GPU) take a
    file lock, so one of them compiles and the others find the library fresh; the compiler
    writes a file of its own, which is renamed into place in one step."""
    lib = out or LIB
    if not force and not _stale(lib):
        return lib
    import fcntl

    with open(lib + ".lock", "w") as lock:
        fcntl.flock(lock, fcntl.LOCK_EX)
        try:
            if not force and not _stale(lib):
                return lib
            nvcc = os.environ.get("NVCC", "nvcc")
            tmp = f"{lib}.tmp{os.getpid()}"
            cmd = [nvcc, *NVCC_FLAGS, *(extra or []), "-I", INCLUDE, *sources(), "-o", tmp]
            if verbose:
                print(" ".join(cmd), flush=True)
            try:
                subprocess.run(cmd, check=True)
                os.replace(tmp, lib)
            finally:
                if os.path.exists(tmp):
                    os.remove(tmp)
        finally:
            fcntl.flock(lock, fcntl.LOCK_UN)
    return lib


if __name__ == "__main__":
    extra = [a for a in sys.argv[1:] if a.startswith("-X")]
    print(build(force=True, verbose=True, extra=["-Xptxas", "-v"] if "-v" in sys.argv else extra))
