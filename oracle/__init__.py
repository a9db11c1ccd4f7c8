"""CPU oracle for the LoopKV decode path.

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the library under
``loop_aware_quantized_b200`` never does, and it shares no code with it.

The arithmetic lives in ``loopkv_oracle.cpp`` (plain C++, fp64 attention,
IEEE fp32 quantization); ``oracle.py`` is a ctypes wrapper around it.
"""

from .oracle import (  # noqa: F401
    KIND_BF16,
    KIND_Q2,
    KIND_Q4,
    KIND_RES2,
    KIND_SHARE,
    DecodeResult,
    OracleUnit,
    decode,
    quantize_group,
    region_bytes,
)
