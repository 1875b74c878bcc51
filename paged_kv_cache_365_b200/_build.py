"""Build libpkv.so in-tree with nvcc for sm_100a.

The library is a plain C-ABI shared object (no torch types), so it is built
with nvcc directly rather than as a torch extension.
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libpkv.so")

SOURCES = ["pkv_api.cu", "allocator.cpp", "plan.cpp"]
HEADERS = ["common.cuh", "decode.cuh", "decode_mma.cuh", "decode_prefix.cuh", "decode_launch.cuh", "decode_fp8.cuh", "multi_mma.cuh", "multi_tc.cuh", "cache_ops.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "pkv.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, extra=None) -> str:
    """Compile the library if any source is newer than it; return its path."""
    if not force and up_to_date():
        return LIB
    cmd = [_nvcc(), "-O3", "-std=c++17", "-lineinfo", *ARCH,
           "-Xcompiler", "-fPIC,-O2,-Wall", "-shared",
           "-I", INCLUDE, "-I", CSRC,
           "-o", LIB + ".tmp"]
    cmd += list(extra or [])
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None)
