"""The input generator's Philox4x32-10 against the published known-answer
vectors of Salmon, Moraes, Dror and Shaw, "Parallel Random Numbers: As Easy
as 1, 2, 3" (SC'11), as distributed with their Random123 library (10 rounds,
four 32-bit counter words, two 32-bit key words).  The host generator is
checked on CPU; its GPU twin, which builds the 16K workloads on the device,
on a B200."""

import numpy as np
import pytest

from synth import philox as px

# (counter c0..c3, key k0, k1) -> output words
KAT = [
    ((0x00000000, 0x00000000, 0x00000000, 0x00000000, 0x00000000, 0x00000000),
     (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
    ((0xFFFFFFFF, 0xFFFFFFFF, 0xFFFFFFFF, 0xFFFFFFFF, 0xFFFFFFFF, 0xFFFFFFFF),
     (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
    ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344, 0xA4093822, 0x299F31D0),
     (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
]


@pytest.mark.parametrize("row, want", KAT)
def test_host_philox_known_answers(row, want):
    got = tuple(int(x) for x in px.philox4x32(*row))
    assert got == want, ["%08x" % x for x in got]


@pytest.mark.gpu
def test_device_philox_known_answers(cuda_device):
    from synth.gpu import philox_rows
    got = philox_rows([r for r, _ in KAT], cuda_device)
    assert np.array_equal(got, np.array([w for _, w in KAT], np.uint32)), got
