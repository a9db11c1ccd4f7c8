"""CUDA path vs CPU oracle on the five seeded workloads (needs a B200).

Packed codes, scales, zero points and low-plane masks must match bit for bit
(mask positions whose oracle weight lies within 1e-6 of tau are exempt);
outputs within 2e-3 absolute and 1e-2 relative (per unit, against the
unit's largest output) of the fp64 oracle; logsumexp within 1e-3.
"""

import numpy as np
import pytest

from synth import workloads as W
from tests import gpu_harness as GH
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pool():
    p = P.make_pool()
    yield p
    p.terminate()


@pytest.fixture(scope="module")
def dev(cuda_device):
    return cuda_device


def _gen(wl, dev):
    from synth.gpu import DeviceGenerator
    return DeviceGenerator(wl, dev)


def test_device_generator_matches_host(dev):
    import torch
    for config in ("0", "2", "2r", "4"):
        wl = W.make(config)
        gen = _gen(wl, dev)
        seqs = [0, wl.batch - 1]
        t0 = np.array([5, 1000], np.int32)
        cells = [0, wl.n_cells - 1]
        if config == "2r":  # a residual cell: its tokens follow its reference's
            cells[0] = int(np.nonzero(wl.kinds == W.RES2)[0][0])
        k, v = gen.kv(cells, seqs, t0, 40)
        kh = k.view(torch.int16).cpu().numpy().view(np.uint16)
        vh = v.view(torch.int16).cpu().numpy().view(np.uint16)
        for ci, c in enumerate(cells):
            for bl, b in enumerate(seqs):
                for h in (0, wl.n_heads - 1):
                    rk = W.raw_keys(wl, c, b, h, int(t0[bl]), int(t0[bl]) + 40)
                    rv = W.raw_values(wl, c, b, h, int(t0[bl]), int(t0[bl]) + 40)
                    assert (kh[ci, bl, h] == rk).all() and (vh[ci, bl, h] == rv).all()
        lens = np.array([[3, 700], [1, 2]], np.int32)
        q = gen.queries(cells, seqs, lens).view(torch.int16).cpu().numpy().view(np.uint16)
        for ci, c in enumerate(cells):
            for bl, b in enumerate(seqs):
                for h in (0, wl.n_heads - 1):
                    assert (q[ci, bl, h] == W.query(wl, c, b, h, int(lens[ci, bl]))).all()
        # query heads of a KV head's group (grouped-query decode)
        qg = gen.queries(cells, seqs, lens, g=3).view(torch.int16).cpu().numpy().view(np.uint16)
        for ci, c in enumerate(cells):
            for bl, b in enumerate(seqs):
                for h in (0, wl.n_heads - 1):
                    ref = W.query_group(wl, c, b, h, int(lens[ci, bl]), 3)
                    assert (qg[ci, bl, h] == ref).all() and (ref[0] == q[ci, bl, h]).all()


def _run_decode_only(config, pool, dev, cells=None, seqs=None, n_sample=16, split=0):
    wl = W.make(config)
    seqs = list(range(wl.batch)) if seqs is None else list(seqs)
    cells = list(range(wl.n_cells)) if cells is None else list(cells)
    # SHARE and RES2 cells need the final loop's cell of their layer as well
    need = sorted(set(cells) | {wl.source_cell(c) for c in cells
                                if wl.kinds[c] in (W.SHARE, W.RES2)})
    lengths = wl.lengths[seqs]
    plan = GH.make_plan(wl, seqs, decode_split=split)
    gen = _gen(wl, dev)
    GH.build_cache(wl, plan, gen, seqs, lengths, cells=need)
    lens = np.array([[wl.lengths[b] for b in seqs] for _ in cells], np.int32)
    res = GH.decode_all(wl, plan, gen, seqs, cells, lens, dev)
    plan.check()
    units = GH.sample_units(wl, cells, seqs, n_sample, seed=int(config[0]) + 7)
    n_of = lambda c, b: int(wl.lengths[b])  # noqa: E731
    stats = GH.compare(config, wl, plan, res, cells, seqs, units, n_of, n_of, pool)
    return stats


def test_config0_tiny_all_units(pool, dev):
    wl = W.make("0")
    units = [(c, 0, h) for c in range(wl.n_cells) for h in range(wl.n_heads)]
    plan = GH.make_plan(wl, [0])
    gen = _gen(wl, dev)
    GH.build_cache(wl, plan, gen, [0], wl.lengths)
    lens = np.full((wl.n_cells, 1), wl.lengths[0], np.int32)
    res = GH.decode_all(wl, plan, gen, [0], list(range(wl.n_cells)), lens, dev)
    n_of = lambda c, b: int(wl.lengths[b])  # noqa: E731
    GH.compare("0", wl, plan, res, list(range(wl.n_cells)), [0], units, n_of, n_of, pool)
    plan.check()


@pytest.mark.parametrize("split", [2, 4, 8])
def test_config0_cluster_split(pool, dev, split):
    _run_decode_only("0", pool, dev, n_sample=8, split=split)


def test_config1_single_sequence(pool, dev):
    _run_decode_only("1", pool, dev, n_sample=24)


def test_config2_batched_16k(pool, dev):
    stats = _run_decode_only("2", pool, dev, n_sample=24)
    assert max(s["max_abs"] for s in stats) < P.OUT_ABS_TOL


def test_config2r_residual_cells_16k(pool, dev):
    # the config-2 plan with its SHARE cells stored as 2-bit residuals
    stats = _run_decode_only("2r", pool, dev, n_sample=24)
    assert max(s["max_abs"] for s in stats) < P.OUT_ABS_TOL


@pytest.mark.parametrize("sub", ["a", "b", "c", "d"])
def test_config3_ablation(pool, dev, sub):
    # every cell of an ablation plan has the same kind: 8 cells of the
    # 16K shape cover it.  The all-bf16 plan (412 GB for the whole batch)
    # runs on a 4-sequence slice of the batch.
    seqs = [0, 9, 22, 31] if sub == "d" else None
    _run_decode_only("3" + sub, pool, dev, cells=[0, 13, 30, 47, 50, 71, 80, 95], seqs=seqs,
                     n_sample=12)


def test_config4_ragged_serving_steps(pool, dev):
    """Ragged batch: bulk build, then steps of one new token per cell in serving
    order (append + decode of loops 0-2, then of loop 3); checked at the last step."""
    import torch
    from loop_aware_quantized_b200 import steps
    wl = W.make("4")
    r = wl.lengths % 32
    # sequences about to flush a group, just flushed, shortest and longest
    pick = [int(np.argmax(r)), int(np.argmin(r)), int(np.argmin(wl.lengths)),
            int(np.argmax(wl.lengths)), 5, 17]
    seqs = sorted(set(pick))
    n0 = wl.lengths[seqs].astype(np.int32)
    plan = GH.make_plan(wl, seqs)
    gen = _gen(wl, dev)
    GH.build_cache(wl, plan, gen, seqs, n0)
    phase = steps.phases(wl.n_loops, wl.n_layers)
    H, D, B = wl.n_heads, wl.head_dim, len(seqs)
    n_steps = 3
    outs = None
    for s in range(n_steps):
        qs, ks, vs, outs, lses, masks, nsels = [], [], [], [], [], [], []
        for i, cells in enumerate(phase):
            k, v = gen.kv(cells, seqs, n0 + s, 1)
            ks.append(k)
            vs.append(v)
            # unit lengths at decode time: n0 + s + 1 for every cell
            lens = np.tile(n0 + s + 1, (len(cells), 1))
            qs.append(gen.queries(cells, seqs, lens))
            shape = (len(cells), B, H)
            outs.append(torch.empty(shape + (D,), dtype=torch.float32, device=dev))
            lses.append(torch.empty(shape, dtype=torch.float32, device=dev))
            masks.append(torch.zeros(shape + (int(wl.capacity.max()) // 32 + 1,),
                                     dtype=torch.int32, device=dev))
            nsels.append(torch.empty(shape, dtype=torch.int32, device=dev))
        steps.decode_step(plan, phase, qs, ks, vs, outs, lse=lses, mask=masks, nsel=nsels)
    torch.cuda.synchronize()
    plan.check()
    assert (plan.lengths()[:, :B] == n0 + n_steps).all()
    nfin = n0 + n_steps
    seqpos = {b: i for i, b in enumerate(seqs)}
    own = lambda c, b: int(nfin[seqpos[b]])  # noqa: E731
    # non-final loops decode before the final loop's append of the same step
    src = lambda c, b: int(nfin[seqpos[b]] - 1)  # noqa: E731
    for i, cells in enumerate(phase):
        res = dict(q=qs[i].view(torch.int16).cpu().numpy().view(np.uint16),
                   out=outs[i].cpu().numpy(), lse=lses[i].cpu().numpy(),
                   nsel=nsels[i].cpu().numpy(), mask=masks[i].cpu().numpy().view(np.uint32))
        units = GH.sample_units(wl, list(cells), seqs, 12, seed=40 + i)
        GH.compare("4", wl, plan, res, list(cells), seqs, units, own, src, pool)
