"""Build libpagedkv.so in-tree with nvcc for sm_100a (B200).

    python -m paged_kv_cache_460_b200.build [--verbose]

The library is a plain shared object with a C ABI (include/pagedkv.h); the Python
binding loads it with ctypes.  nvcc cross-compiles, so this runs without a GPU.
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libpagedkv.so")
SOURCES = ["pagedkv.cu", "pool.cpp"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _inputs():
    names = os.listdir(CSRC)
    files = [os.path.join(CSRC, n) for n in names if n.endswith((".cu", ".cuh", ".cpp", ".h"))]
    return files + [os.path.join(INCLUDE, "pagedkv.h"), os.path.abspath(__file__)]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, out: str = None, defines=()) -> str:
    """Compile the library (to `out`, default in-tree) unless it is up to date."""
    lib = out or LIB
    if not force and out is None and not defines and up_to_date():
        return LIB
    tmp = lib + ".tmp.%d" % os.getpid()
    cmd = [NVCC, "-O3", "-std=c++17", *ARCH, "-lineinfo", "-shared", "-Xcompiler", "-fPIC",
           "-I", INCLUDE, "-I", CSRC, "-o", tmp] + ["-D" + d for d in defines]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libpagedkv.so")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
