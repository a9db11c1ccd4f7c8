"""Write the oracle's golden values (``oracle_golden.json``).

Calls only the CPU oracle (``oracle/``) and the seeded input generator
(``synth/``).  The stored values pin the oracle against unintended changes:
``tests/test_golden_cpu.py`` recomputes them.  A change to the oracle's
arithmetic that moves them is regenerated with this script, and its commit
names the passage of the pages (or the reading of it) that justifies it.

Cases: the 2 loops x 2 layers tiny workload (4-bit, SHARE, 2-bit, 4-bit
cells; "LoopKV: Loop-Aware KV Cache Compression for Serving Looped
Transformers", section 概要), the same plan with its SHARE cell stored as a
RES2 cell (ResidualQuant, as summarised in the related-paper list of the
page "LoopVQ: Sub 1-bit KV Cache Quantization for Looped Transformers"),
and a LoopVQ unit ("LoopVQ: ...", section 概要).

Run: python tests/golden/make_golden.py
"""

import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

from oracle import oracle as orc  # noqa: E402
from synth import workloads as W  # noqa: E402
from tests import parity as P  # noqa: E402

RES2_SPEC = (2, 2, 2, 64, (W.Q4, W.RES2, W.Q2, W.Q4), (256,), (320,), 0.01)


def unit_record(config, cell, h):
    wl = P.workload(config)
    n = int(wl.lengths[0])
    ref = P.oracle_unit_job((config, cell, 0, h, n, n, False))
    return {"cell": cell, "head": h, "kind": W.KIND_NAMES[ref["kind"]],
            "out": [float(x) for x in ref["out"]], "lse": float(ref["lse"]),
            "mask": [int(x) for x in ref["mask"]], "nsel": int(ref["nsel"])}


def golden():
    tiny = [unit_record("0", c, h) for c in range(4) for h in range(2)]
    res2 = [unit_record(RES2_SPEC, 1, h) for h in range(2)]
    wv = W.make_vq("vqsmall")
    vq = []
    for loop, layer, b, h in ((0, 0, 2, 1), (3, 1, 1, 0)):
        n = int(wv.lengths[b])
        out, lse = orc.vq_decode(W.vq_indices(wv, 0, layer, b, h, 0, n),
                                 W.vq_indices(wv, 1, layer, b, h, 0, n),
                                 W.vq_codebook(wv, 0, layer, h), W.vq_codebook(wv, 1, layer, h),
                                 W.vq_query(wv, loop, layer, b, h), loop, wv.n_loops)
        vq.append({"loop": loop, "layer": layer, "seq": b, "head": h,
                   "out": [float(x) for x in out], "lse": float(lse)})
    return {"tiny": tiny, "res2": res2, "vq": vq}


if __name__ == "__main__":
    with open(os.path.join(HERE, "oracle_golden.json"), "w") as f:
        json.dump(golden(), f, indent=0)
    print("wrote", os.path.join(HERE, "oracle_golden.json"))
