"""Build the CPU oracle (oracle/liboracle.so) with gcc.  Test infrastructure only."""

from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-fPIC",
           "-shared", SRC, "-o", LIB, "-lm"]
    subprocess.run(cmd, check=True)
    return LIB


LIB_OMP = os.path.join(HERE, "liboracle_omp.so")


def build_omp(force: bool = False) -> str:
    """The same oracle.c with -fopenmp: its token loops run on all host cores.  Only the
    benchmark's CPU-baseline leg uses it, to report the oracle's multi-core time."""
    if not force and os.path.exists(LIB_OMP) and os.path.getmtime(LIB_OMP) >= os.path.getmtime(SRC):
        return LIB_OMP
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-fPIC", "-fopenmp",
           "-shared", SRC, "-o", LIB_OMP, "-lm"]
    subprocess.run(cmd, check=True)
    return LIB_OMP


def build_variant(source: str, lib_path: str) -> str:
    """Compile another version of oracle.c (given as text) to `lib_path`."""
    src = lib_path + ".c"
    with open(src, "w") as f:
        f.write(source)
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-fPIC",
                    "-shared", src, "-o", lib_path, "-lm"], check=True)
    return lib_path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
    print(build_omp(force="--force" in sys.argv))
