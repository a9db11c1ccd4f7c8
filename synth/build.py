"""Build the GPU input generator ``synth/libloopkv_synth.so`` (sm_100a)."""

import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "synth.cu")
LIB = os.path.join(HERE, "libloopkv_synth.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-Xcompiler", "-fPIC",
         "-shared"]


def _stamp():
    """Hash of the source, the flags and the compiler's version text."""
    h = hashlib.sha256()
    with open(SRC, "rb") as f:
        h.update(f.read())
    h.update(" ".join(FLAGS).encode())
    h.update(subprocess.run([NVCC, "--version"], capture_output=True, check=True).stdout)
    return h.hexdigest()


def build(force=False):
    """Build unless the library exists with a stamp (libloopkv_synth.so.stamp)
    matching the current source, flags and compiler."""
    stamp = _stamp()
    stamp_path = LIB + ".stamp"
    if not force and os.path.exists(LIB) and os.path.exists(stamp_path):
        with open(stamp_path) as f:
            if f.read().strip() == stamp:
                return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    subprocess.check_call([NVCC, *FLAGS, SRC, "-o", tmp, "-cudart", "static"])
    os.replace(tmp, LIB)
    with open(stamp_path, "w") as f:
        f.write(stamp + "\n")
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
