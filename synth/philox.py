"""Counter-based random numbers for the synthetic inputs (host side).

Philox4x32-10 as published in Salmon, Moraes, Dror and Shaw, "Parallel Random
Numbers: As Easy as 1, 2, 3" (SC'11): a 128-bit counter and a 64-bit key go
through ten rounds of two 32x32->64 multiplies, with the key bumped by the
Weyl constants between rounds.  ``synth/csrc/synth.cu`` implements the same
definition on the GPU; the two agree bit for bit, so any slice of a workload
the GPU generates can be regenerated here.

This module holds no LoopKV arithmetic: it only turns counters into bits,
bits into approximately normal fp32 values, and fp32 into bf16 bit patterns.
"""

import numpy as np

M0 = np.uint64(0xD2511F53)
M1 = np.uint64(0xCD9E8D57)
W0 = np.uint32(0x9E3779B9)
W1 = np.uint32(0xBB67AE85)
MASK32 = np.uint64(0xFFFFFFFF)

# Standard deviation of a sum of eight independent uniform draws on
# {0, ..., 65535}; NORMAL_SCALE maps that sum (centred) to unit variance.
NORMAL_CENTER = 8 * 65535 // 2  # 262140
NORMAL_SCALE = np.float32(1.0 / np.sqrt(8.0 * (65536.0 ** 2 - 1.0) / 12.0))


def philox4x32(c0, c1, c2, c3, k0, k1):
    """Philox4x32-10 of broadcastable uint32 counters and a (k0, k1) key.

    Returns four uint32 arrays.
    """
    c0, c1, c2, c3 = (np.asarray(c, dtype=np.uint32) for c in (c0, c1, c2, c3))
    c0, c1, c2, c3 = np.broadcast_arrays(c0, c1, c2, c3)
    c0, c1, c2, c3 = (c.astype(np.uint32, copy=True) for c in (c0, c1, c2, c3))
    k0 = np.uint32(k0)
    k1 = np.uint32(k1)
    with np.errstate(over="ignore"):
        for r in range(10):
            if r:
                k0 = np.uint32(k0 + W0)
                k1 = np.uint32(k1 + W1)
            p0 = M0 * c0.astype(np.uint64)
            p1 = M1 * c2.astype(np.uint64)
            hi0 = (p0 >> np.uint64(32)).astype(np.uint32)
            lo0 = (p0 & MASK32).astype(np.uint32)
            hi1 = (p1 >> np.uint64(32)).astype(np.uint32)
            lo1 = (p1 & MASK32).astype(np.uint32)
            c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return c0, c1, c2, c3


def normal_from_bits(u0, u1, u2, u3):
    """Approximately N(0,1) fp32 from four uint32 words.

    Sum of the eight 16-bit halves (an Irwin-Hall sum of eight uniforms),
    centred and scaled to unit variance.  Integer sum, one exact int->fp32
    conversion and one fp32 multiply: bit-exact on any IEEE machine.  The
    tails are cut at about 4.9 standard deviations.
    """
    s = np.zeros(np.shape(u0), dtype=np.int64)
    for u in (u0, u1, u2, u3):
        u = np.asarray(u, dtype=np.uint32).astype(np.int64)
        s += (u & 0xFFFF) + (u >> 16)
    d = (s - NORMAL_CENTER).astype(np.float32)
    return (d * NORMAL_SCALE).astype(np.float32)


def uniform_index(u, n):
    """floor(u * n / 2**32) for uint32 u and integer n >= 1 (exact)."""
    return ((np.asarray(u, dtype=np.uint64) * np.uint64(n)) >> np.uint64(32)).astype(np.int64)


def float_to_bf16_bits(x):
    """Round fp32 to bf16 (nearest, ties to even) and return the bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_float(b):
    """bf16 bit patterns -> fp32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)
