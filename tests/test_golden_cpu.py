"""The CPU oracle against its stored golden values (``tests/golden``, written
by ``tests/golden/make_golden.py`` from the oracle itself): any change of
the oracle's results shows up here.  CPU only."""

import json
import os

import numpy as np

from tests.golden import make_golden as MG

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_oracle_matches_its_golden_values():
    with open(os.path.join(HERE, "oracle_golden.json")) as f:
        stored = json.load(f)
    now = MG.golden()
    for part in ("tiny", "res2", "vq"):
        assert len(now[part]) == len(stored[part]), part
        for a, b in zip(now[part], stored[part]):
            assert np.abs(np.array(a["out"]) - np.array(b["out"])).max() < 1e-12, (part, b)
            assert abs(a["lse"] - b["lse"]) < 1e-12, (part, b)
            for key in ("mask", "nsel", "kind"):
                if key in b:
                    assert a[key] == b[key], (part, key, b)
