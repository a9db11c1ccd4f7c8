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
OUT_REL_TOL = 1e-2      # relative error, in two forms (check_unit):
                        #   per head, max_d |diff| / max(max_d |out_oracle|, 1e-6), and
                        #   per element, |diff| / |out_oracle| where |out_oracle| >= REL_FLOOR
REL_FLOOR = 0.05        # below it the absolute bound is the binding one: 1e-2 x 0.05 is
                        # already 4x tighter than OUT_ABS_TOL
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

    args = (config, cell, b, h, n_own, n_src, g[, sel_override]).  Returns the
    host query bits [g][D] and the oracle's per-head outputs, union mask and
    count.  ``sel_override``: mask words deciding the positions within BAND of
    tau (the kernel's choice there)."""
    from oracle import oracle as orc
    config, cell, b, h, n_own, n_src, g = args[:7]
    override = args[7] if len(args) > 7 else None
    wl = workload(config)
    own, src = _oracle_units(orc, wl, cell, b, n_own, n_src, h)
    q = W.query_group(wl, cell, b, h, n_own, g)
    r = orc.decode_group(own, q, wl.tau, src=src, band=BAND, sel_override=override)
    return dict(q=q, out=r.out, lse=r.lse, mask=r.mask, nsel=r.nsel, weights=r.weights,
                kind=int(wl.kinds[cell]), job=tuple(args[:7]), group=True)


def oracle_unit_job(args):
    """Build the oracle state of one unit and decode it.

    args = (config, cell, b, h, n_own, n_src, want_bytes[, sel_override]):
    n_own tokens in the unit, n_src tokens in its SHARE source or RES2
    reference (ignored otherwise); ``sel_override`` as in oracle_group_job.
    Returns a dict with the host query bits, the oracle result and, if asked,
    the unit's canonical bytes.
    """
    from oracle import oracle as orc
    config, cell, b, h, n_own, n_src, want_bytes = args[:7]
    override = args[7] if len(args) > 7 else None
    wl = workload(config)
    kind = int(wl.kinds[cell])
    own, src = _oracle_units(orc, wl, cell, b, n_own, n_src, h)
    q = W.query(wl, cell, b, h, n_own)
    r = orc.decode(own, q, wl.tau, src=src, band=BAND, sel_override=override)
    out = dict(q=q, out=r.out, lse=r.lse, mask=r.mask, nsel=r.nsel, weights=r.weights,
               kind=kind, job=(config, cell, b, h, n_own, n_src, False), group=False)
    if want_bytes:
        out["bytes"], out["valid"] = own.serialize(src=src if kind == W.RES2 else None)
    return out


def make_pool(workers=None):
    ctx = mp.get_context("spawn")
    n = workers or max(1, min(32, (os.cpu_count() or 2) - 1))
    return ctx.Pool(n)


# ------------------------------------------------------------- comparisons

def exempt_bits(weights, n_words, tau):
    """Mask words with a bit set for positions whose oracle weight (of any
    head: weights [npos] or [g][npos]) is within BAND of tau."""
    w = np.atleast_2d(np.asarray(weights))[:, : n_words * G]
    ex = np.zeros(n_words, np.uint32)
    near = np.nonzero((np.abs(w - tau) <= BAND).any(axis=0))[0]
    for pos in near:
        ex[pos // G] |= np.uint32(1) << np.uint32(pos % G)
    return ex


def recompute_with(ref, gpu_mask):
    """The oracle's result for ref's unit with the kernel's selection on the
    positions within BAND of tau (the only ones where the two may differ)."""
    words = np.asarray(gpu_mask, np.uint32)[: len(ref["mask"])].copy()
    job = tuple(ref["job"]) + (words,)
    return oracle_group_job(job) if ref["group"] else oracle_unit_job(job)


def check_unit(tag, ref, out, lse=None, mask=None, nsel=None, tau=0.0):
    """Assert one unit's GPU results against its oracle result; returns stats.

    ``out``: [D] (one query) or [g][D] (a query group); ``lse`` likewise.
    Masks must agree bit for bit outside the BAND around tau.  Where the
    kernel chose differently on a position inside the band, the oracle is
    recomputed with the kernel's choice there, so the outputs are compared at
    the full tolerance; that needs the kernel's mask whenever the unit has
    such positions."""
    n_exempt = 0
    if "mask" in ref and len(ref["mask"]):
        words = len(ref["mask"])
        ex = exempt_bits(ref["weights"], words, tau)
        n_exempt = int(sum(bin(int(x)).count("1") for x in ex))
        if mask is None:
            assert n_exempt == 0, "%s: %d positions within the band of tau; pass the kernel's mask" % (
                tag, n_exempt)
        else:
            gm = np.asarray(mask[:words]).astype(np.uint32)
            diff = gm ^ ref["mask"]
            assert (diff & ~ex == 0).all(), "%s: mask differs in words %s" % (
                tag, np.nonzero(diff & ~ex)[0][:8])
            if diff.any():
                ref = recompute_with(ref, gm)
                assert np.array_equal(ref["mask"], gm), tag + ": override did not take"
    if nsel is not None:
        assert int(nsel) == ref["nsel"], "%s: nsel %d vs %d" % (tag, nsel, ref["nsel"])
    want = np.asarray(ref["out"], np.float64)
    got = np.asarray(out, np.float64).reshape(want.shape)
    err = np.abs(got - want)
    assert (err <= OUT_ABS_TOL).all(), "%s: max abs err %.3g" % (tag, err.max())
    w2, e2 = np.atleast_2d(want), np.atleast_2d(err)
    scale = np.maximum(np.abs(w2).max(axis=1), 1e-6)
    rel = (e2.max(axis=1) / scale).max()
    assert rel <= OUT_REL_TOL, "%s: rel err %.3g" % (tag, rel)
    big = np.abs(want) >= REL_FLOOR
    if big.any():
        rel_el = (err[big] / np.abs(want[big])).max()
        assert rel_el <= OUT_REL_TOL, "%s: element rel err %.3g" % (tag, rel_el)
    if lse is not None:
        got_l = np.asarray(lse, np.float64).reshape(-1)
        want_l = np.asarray(ref["lse"], np.float64).reshape(-1)
        assert (np.abs(got_l - want_l) <= LSE_TOL + 1e-5 * np.abs(want_l)).all(), (
            "%s: lse %s vs %s" % (tag, got_l, want_l))
    return dict(max_abs=float(err.max()), max_rel=float(rel), exempt=n_exempt)


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
