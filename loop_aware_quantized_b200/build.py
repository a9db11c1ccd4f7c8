"""Build the LoopKV CUDA library in-tree for sm_100a.

Produces ``loop_aware_quantized_b200/libloopkv.so`` from ``csrc/*.cu`` with
nvcc (``-gencode arch=compute_100a,code=sm_100a``).  Runs without a GPU.
"""

import glob
import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libloopkv.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    # decode converts codes to floats as exact subnormals: keep them
    "-ftz=false", "-prec-div=true", "-prec-sqrt=true",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [
        os.path.join(ROOT, "include", "loopkv.h")]


def _stamp(flags):
    """Hash of what the library is built from: every source and header, the
    flags and the compiler's version text."""
    h = hashlib.sha256()
    for d in _deps():
        h.update(os.path.relpath(d, ROOT).encode())
        with open(d, "rb") as f:
            h.update(f.read())
    h.update(" ".join(flags).encode())
    h.update(subprocess.run([NVCC, "--version"], capture_output=True, check=True).stdout)
    return h.hexdigest()


def build(force=False, verbose=False, extra_flags=()):
    """Compile libloopkv.so unless it exists with a stamp matching the current
    sources, flags and compiler (kept in libloopkv.so.stamp beside it)."""
    flags = [*NVCC_FLAGS, *extra_flags]
    stamp = _stamp(flags)
    stamp_path = LIB + ".stamp"
    if not force and os.path.exists(LIB) and os.path.exists(stamp_path):
        with open(stamp_path) as f:
            if f.read().strip() == stamp:
                return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = [NVCC, *flags, "-shared", "-I", os.path.join(ROOT, "include"),
           *sources(), "-o", tmp, "-cudart", "static"]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    with open(stamp_path, "w") as f:
        f.write(stamp + "\n")
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True,
                extra_flags=["-Xptxas", "-v"] if "--ptxas" in sys.argv else []))
