"""The parity harness on CPU: when the kernel decides a position whose
weight lies within the band around tau differently from the oracle, the
harness recomputes the oracle with the kernel's choice there and compares the
outputs at the full tolerance; any other disagreement fails.  The "kernel"
results here are the oracle's own, with one such position decided the other
way, so no GPU is needed."""

import numpy as np
import pytest

from synth import workloads as W
from tests import parity as P


def _near_tau_unit():
    """A 4-bit unit and a tau equal to the weight of one of its quantized
    positions (a mid-weight one), so that position sits inside the band."""
    base = (2, 2, 2, 64, (W.Q4, W.Q2, W.Q2, W.Q4), (200,), (256,), 0.01)
    job = (base, 0, 0, 1, 200, 200, False)
    ref = P.oracle_unit_job(job)
    w = ref["weights"][:192]
    t = int(np.argsort(w)[-4])
    spec = base[:7] + (float(w[t]),)
    return spec, t


def test_kernel_choice_inside_the_band_is_reproduced():
    spec, t = _near_tau_unit()
    tau = spec[7]
    ref = P.oracle_unit_job((spec, 0, 0, 1, 200, 200, False))
    assert (ref["mask"][t // 32] >> (t % 32)) & 1            # p == tau: selected
    flipped = ref["mask"].copy()
    flipped[t // 32] ^= np.uint32(1 << (t % 32))
    kern = P.oracle_unit_job((spec, 0, 0, 1, 200, 200, False, flipped))
    assert kern["nsel"] == ref["nsel"] - 1
    moved = np.abs(kern["out"] - ref["out"]).max()
    assert moved > 0.0
    st = P.check_unit("flipped", ref, kern["out"].astype(np.float32), lse=ref["lse"],
                      mask=kern["mask"], nsel=kern["nsel"], tau=tau)
    assert st["exempt"] >= 1 and st["max_abs"] < 1e-6       # compared against the recomputed oracle


def test_disagreements_that_are_not_allowed_fail():
    spec, t = _near_tau_unit()
    tau = spec[7]
    ref = P.oracle_unit_job((spec, 0, 0, 1, 200, 200, False))
    out = ref["out"].astype(np.float32)
    # a selected position far from tau reported as not selected
    far = int(np.argmax(ref["weights"][:192]))
    bad = ref["mask"].copy()
    bad[far // 32] ^= np.uint32(1 << (far % 32))
    with pytest.raises(AssertionError, match="mask differs"):
        P.check_unit("far", ref, out, mask=bad, nsel=ref["nsel"] - 1, tau=tau)
    # a count that does not match the mask
    with pytest.raises(AssertionError, match="nsel"):
        P.check_unit("count", ref, out, mask=ref["mask"], nsel=ref["nsel"] + 1, tau=tau)
    # an output off by more than the absolute bound
    off = out.copy()
    off[3] += 3e-3
    with pytest.raises(AssertionError, match="abs err"):
        P.check_unit("abs", ref, off, mask=ref["mask"], nsel=ref["nsel"], tau=tau)
    # a unit with a position inside the band cannot be checked without the kernel's mask
    with pytest.raises(AssertionError, match="within the band"):
        P.check_unit("no mask", ref, out, tau=tau)


def test_element_relative_error_is_checked():
    spec, t = _near_tau_unit()
    ref = P.oracle_unit_job((spec, 0, 0, 1, 200, 200, False))
    out = ref["out"].astype(np.float64).copy()
    big = np.nonzero(np.abs(out) >= P.REL_FLOOR)[0]
    small = big[np.argmin(np.abs(out[big]))]
    # within the absolute bound, beyond 1e-2 of that element
    out[small] += np.sign(out[small]) * min(1.5e-3, 0.02 * abs(out[small]))
    if abs(out[small] - ref["out"][small]) / abs(ref["out"][small]) <= P.OUT_REL_TOL:
        pytest.skip("no element small enough to separate the two bounds")
    with pytest.raises(AssertionError, match="rel err"):
        P.check_unit("rel", ref, out, mask=ref["mask"], nsel=ref["nsel"], tau=spec[7])
