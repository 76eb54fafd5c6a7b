"""Compile the fp64 CPU oracle (oracle.c) with gcc: oracle/liboracle.so, and
oracle/liboracle_omp.so, the same source built with OpenMP so that the (sequence, head)
pair routines run their independent pairs on all host cores (the CPU baseline's all-core
leg).  The arithmetic of every pair is identical in both builds.

Test infrastructure: the oracle is the checker, not part of the product.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")
LIB_OMP = os.path.join(HERE, "liboracle_omp.so")


def build(force: bool = False, omp: bool = False) -> str:
    """Build the plain (or OpenMP) library when it is missing or older than oracle.c;
    return its path."""
    lib = LIB_OMP if omp else LIB
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= os.path.getmtime(SRC):
        return lib
    tmp = lib + ".tmp.%d" % os.getpid()
    # -O2 only: no -ffast-math, so the fp64 arithmetic keeps IEEE semantics and order.
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off"]
    cmd += ["-fopenmp"] if omp else []
    cmd += ["-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build_all(force: bool = False):
    return build(force), build(force, omp=True)


if __name__ == "__main__":
    print(build_all(force=True))
