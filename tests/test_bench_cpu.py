"""bench.py's host logic without a GPU: the decode byte model (the
roofline's numerator) against the bytes the oracle's canonical layout
stores, and the reference arm's JSON line."""

import json
import os
import subprocess
import sys

import numpy as np
import pytest

from synth import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
Q4, Q2, SH, BF, RS = W.Q4, W.Q2, W.SHARE, W.BF16, W.RES2


def _unit(orc, kind, D, n, cap=256):
    """An oracle unit holding n zero tokens (the layout does not depend on values)."""
    u = orc.OracleUnit(kind, D, cap)
    if n:
        z = np.zeros((n, D), np.uint16)
        u.append(z, z)
    return u


def _stored(orc, kind, D, n, src=None):
    """Bytes a decode of the unit streams, from the oracle's layout: every
    byte its serialisation defines, less the 4-bit low value plane, which a
    decode reads per selected token only."""
    u = _unit(orc, kind, D, n)
    _, valid = u.serialize(src=src)
    lo = u.export(src=src)["qtok"] * (D // 4) if kind == Q4 else 0
    return int(valid.sum()) - lo


@pytest.mark.parametrize("D", [64, 128])
def test_decode_byte_model_matches_the_layout(D):
    import bench
    from oracle import oracle as orc
    qo = 2 * D + 4 * D  # the query read and the output written, per unit
    for kind in (Q4, Q2, BF):
        for n in (1, 31, 32, 33, 64, 100, 255):
            wl = W.custom(1, 1, 1, D, (kind,), (n,), (256,), 0.01)
            model = bench.decode_bytes(wl, [0], [n], [n], 0)
            assert model - qo == _stored(orc, kind, D, n), (kind, n)
            # selected tokens add their low-plane row
            assert bench.decode_bytes(wl, [0], [n], [n], 7) == model + 7 * (D // 4)
    # SHARE over a 4-bit source: the source's n - 1 positions as stored, plus
    # the SHARE cell's own current token
    for n in (1, 33, 65, 200):
        wl = W.custom(2, 1, 1, D, (SH, Q4), (n,), (256,), 0.01)
        model = bench.decode_bytes(wl, [0], [n], [n - 1], 0)
        assert model - qo == _stored(orc, Q4, D, n - 1) + _stored(orc, SH, D, n), n
    # RES2 over a fully quantized 4-bit reference: its residual-coded
    # positions read the reference's bytes and its own; the window is bf16
    ref_tokens = 256
    ref = _unit(orc, Q4, D, ref_tokens)
    per_ref_token = _stored(orc, Q4, D, ref_tokens) / ref_tokens
    for n in (1, 63, 64, 65, 130, 200):
        wl = W.custom(2, 1, 1, D, (RS, Q4), (n,), (256,), 0.01)
        model = bench.decode_bytes(wl, [0], [n], [n], 0)
        rt = _unit(orc, RS, D, n).export(src=ref)["qtok"]   # residual-coded positions
        assert model - qo == _stored(orc, RS, D, n, src=ref) + rt * per_ref_token, n


def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "0",
                        "--steps", "2", "--warmup", "1", "--cpu-seconds", "1"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "cell-steps/s" and d["value"] > 0
    assert d["steps"] == 2 and d["warmup"] == 1 and d["higher_is_better"] is True
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
