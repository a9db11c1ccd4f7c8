"""Helpers for comparing the CUDA path with the CPU oracle on seeded inputs.

Oracle inputs come only from the host generator (``synth``); expected values
come only from ``oracle``.  Per-unit oracle work runs in a process pool that
is started with ``spawn`` before the first GPU call.
"""

import functools
import multiprocessing as mp
import os

import numpy as np

from synth import philox as px
from synth import workloads as W

G = 32
OUT_ABS_TOL = 2e-3      # max |out_gpu - out_oracle| per element
OUT_REL_TOL = 1e-2      # max_d |diff| / max(max_d |out_oracle|, 1e-6) per unit
LSE_TOL = 1e-3          # natural-log logsumexp, absolute (+1e-5 relative)
BAND = 1e-6             # mask tokens with |p - tau| <= BAND are exempt


@functools.lru_cache(maxsize=16)
def workload(config):
    """Workload of a config name, or of a hashable ``W.custom`` argument tuple."""
    if isinstance(config, tuple):
        return W.custom(*config)
    return W.make(config)


def _oracle_units(orc, wl, cell, b, n_own, n_src, h):
    """The oracle's unit (and the SHARE source or RES2 reference: the final
    loop's unit, n_src tokens) for (cell, b, h), built from the host
    generator's raw keys and values."""
    kind = int(wl.kinds[cell])
    cap = int(wl.capacity[b])
    own = orc.OracleUnit(kind, wl.head_dim, cap)
    if kind == W.SHARE:
        # A SHARE unit keeps only its current token; earlier tokens only add
        # to its length, so they are appended as zeros.
        k = np.zeros((n_own, wl.head_dim), np.uint16)
        v = np.zeros((n_own, wl.head_dim), np.uint16)
        k[-1] = W.raw_keys(wl, cell, b, h, n_own - 1, n_own)[0]
        v[-1] = W.raw_values(wl, cell, b, h, n_own - 1, n_own)[0]
        own.append(k, v)
        src_cell = wl.source_cell(cell)
        src = orc.OracleUnit(int(wl.kinds[src_cell]), wl.head_dim, cap)
        src.append(W.raw_keys(wl, src_cell, b, h, 0, n_src), W.raw_values(wl, src_cell, b, h, 0, n_src))
    else:
        own.append(W.raw_keys(wl, cell, b, h, 0, n_own), W.raw_values(wl, cell, b, h, 0, n_own))
        src = None
        if kind == W.RES2:
            src_cell = wl.source_cell(cell)
            src = orc.OracleUnit(int(wl.kinds[src_cell]), wl.head_dim, cap)
            src.append(W.raw_keys(wl, src_cell, b, h, 0, n_src),
                       W.raw_values(wl, src_cell, b, h, 0, n_src))
    return own, src


def oracle_group_job(args):
    """Oracle decode of one KV unit for its group of g query heads.

    args = (config, cell, b, h, n_own, n_src, g).  Returns the host query
    bits [g][D] and the oracle's per-head outputs, union mask and count."""
    from oracle import oracle as orc
    config, cell, b, h, n_own, n_src, g = args
    wl = workload(config)
    own, src = _oracle_units(orc, wl, cell, b, n_own, n_src, h)
    q = W.query_group(wl, cell, b, h, n_own, g)
    r = orc.decode_group(own, q, wl.tau, src=src, band=BAND)
    return dict(q=q, out=r.out, lse=r.lse, mask=r.mask, nsel=r.nsel, slack=r.slack,
                weights=r.weights, kind=int(wl.kinds[cell]))


def oracle_unit_job(args):
    """Build the oracle state of one unit and decode it.

    args = (config, cell, b, h, n_own, n_src, want_bytes): n_own tokens in the
    unit, n_src tokens in its SHARE source or RES2 reference (ignored
    otherwise).
    Returns a dict with the host query bits, the oracle result and, if asked,
    the unit's canonical bytes.
    """
    from oracle import oracle as orc
    config, cell, b, h, n_own, n_src, want_bytes = args
    wl = workload(config)
    kind = int(wl.kinds[cell])
    own, src = _oracle_units(orc, wl, cell, b, n_own, n_src, h)
    q = W.query(wl, cell, b, h, n_own)
    r = orc.decode(own, q, wl.tau, src=src, band=BAND)
    out = dict(q=q, out=r.out, lse=r.lse, mask=r.mask, nsel=r.nsel, slack=r.slack,
               weights=r.weights, kind=kind)
    if want_bytes:
        out["bytes"], out["valid"] = own.serialize(src=src if kind == W.RES2 else None)
    return out


def make_pool(workers=None):
    ctx = mp.get_context("spawn")
    n = workers or max(1, min(32, (os.cpu_count() or 2) - 1))
    return ctx.Pool(n)


# ------------------------------------------------------------- comparisons

def exempt_bits(weights, n_words, tau):
    """Mask words with a bit set for positions whose oracle weight is within BAND of tau."""
    ex = np.zeros(n_words, np.uint32)
    near = np.nonzero(np.abs(weights[: n_words * G] - tau) <= BAND)[0]
    for pos in near:
        ex[pos // G] |= np.uint32(1) << np.uint32(pos % G)
    return ex


def check_unit(tag, ref, out, lse=None, mask=None, nsel=None, tau=0.0):
    """Assert one unit's GPU results against its oracle result; returns stats."""
    err = np.abs(out.astype(np.float64) - ref["out"])
    over = np.maximum(err - ref["slack"], 0.0)
    assert (over <= OUT_ABS_TOL).all(), "%s: max abs err %.3g (slack %.3g)" % (
        tag, err.max(), ref["slack"].max())
    scale = max(np.abs(ref["out"]).max(), 1e-6)
    assert over.max() / scale <= OUT_REL_TOL, "%s: rel err %.3g" % (tag, over.max() / scale)
    n_exempt = 0
    if mask is not None:
        words = len(ref["mask"])
        ex = exempt_bits(ref["weights"], words, tau)
        diff = (mask[:words].astype(np.uint32) ^ ref["mask"]) & ~ex
        assert (diff == 0).all(), "%s: mask differs in words %s" % (tag, np.nonzero(diff)[0][:8])
        n_exempt = int(sum(bin(int(x)).count("1") for x in ex))
    if nsel is not None:
        assert abs(int(nsel) - ref["nsel"]) <= n_exempt, "%s: nsel %d vs %d" % (tag, nsel, ref["nsel"])
    if lse is not None:
        assert abs(float(lse) - ref["lse"]) <= LSE_TOL + 1e-5 * abs(ref["lse"]), (
            "%s: lse %.6f vs %.6f" % (tag, lse, ref["lse"]))
    return dict(max_abs=float(err.max()), max_rel=float(err.max() / scale), exempt=n_exempt)


def check_bytes(tag, ref, gpu_bytes):
    """Bit-exact comparison of a unit's cache region over the bytes the oracle defines."""
    valid = ref["valid"].astype(bool)
    g = np.asarray(gpu_bytes)
    assert g.shape == ref["bytes"].shape, "%s: region %s vs %s" % (tag, g.shape, ref["bytes"].shape)
    bad = np.nonzero((g != ref["bytes"]) & valid)[0]
    assert bad.size == 0, "%s: %d cache bytes differ, first at %d" % (tag, bad.size, bad[0])


def bits_to_bf16_tensor(bits, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).view(
        torch.bfloat16).to(device)
