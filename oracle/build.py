"""Compile the CPU oracle into ``oracle/liboracle.so``.

Test infrastructure: plain g++, no fast-math and no floating-point contraction
so that every fp32 step of the quantizer is the IEEE round-to-nearest one.
"""

import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "loopkv_oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")

FLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-Wall",
         "-shared", "-fPIC"]


def _stamp():
    """Hash of the source, the flags and the compiler's version text."""
    h = hashlib.sha256()
    with open(SRC, "rb") as f:
        h.update(f.read())
    h.update(" ".join(FLAGS).encode())
    h.update(subprocess.run(["g++", "--version"], capture_output=True, check=True).stdout)
    return h.hexdigest()


def build(force: bool = False) -> str:
    """Build the oracle library unless it exists with a stamp (liboracle.so.stamp)
    matching the current source, flags and compiler."""
    stamp = _stamp()
    stamp_path = LIB + ".stamp"
    if not force and os.path.exists(LIB) and os.path.exists(stamp_path):
        with open(stamp_path) as f:
            if f.read().strip() == stamp:
                return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    subprocess.check_call(["g++", *FLAGS, SRC, "-o", tmp])
    os.replace(tmp, LIB)
    with open(stamp_path, "w") as f:
        f.write(stamp + "\n")
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
