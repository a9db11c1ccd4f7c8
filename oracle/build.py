"""Compile the CPU oracle into ``oracle/liboracle.so``.

Test infrastructure: plain g++, no fast-math and no floating-point contraction
so that every fp32 step of the quantizer is the IEEE round-to-nearest one.
"""

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "loopkv_oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")

FLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-Wall",
         "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Build the oracle library if missing or older than its source."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    subprocess.check_call(["g++", *FLAGS, SRC, "-o", tmp])
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
