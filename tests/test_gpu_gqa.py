"""Grouped-query decode on the CUDA path (several query heads per KV head)
against the CPU oracle's group decode (needs a B200): every head's output
and logsumexp, and the KV head's union mask and count."""

import numpy as np
import pytest

from synth import workloads as W
from tests import gpu_harness as GH
from tests import parity as P

pytestmark = pytest.mark.gpu

Q4, Q2, SH, BF = W.Q4, W.Q2, W.SHARE, W.BF16


@pytest.fixture(scope="module")
def pool():
    p = P.make_pool(8)
    yield p
    p.terminate()


def _spec(D, kinds, lengths, tau, H=2, extra=64):
    cap = tuple(int((n + extra + 31) // 32 * 32) for n in lengths)
    return (2, 2, H, D, tuple(kinds), tuple(lengths), cap, tau)


def _run(spec, g, pool, dev, split=0):
    """Build every cell, decode every unit for its g query heads, oracle-check all."""
    import torch
    from loop_aware_quantized_b200 import Plan
    from synth.gpu import DeviceGenerator
    wl = W.custom(*spec)
    seqs = list(range(wl.batch))
    plan = Plan(wl.n_loops, wl.n_layers, wl.n_heads, wl.head_dim, wl.capacity[seqs], wl.kinds,
                wl.tau, q_per_kv=g, decode_split=split)
    gen = DeviceGenerator(wl, dev)
    GH.build_cache(wl, plan, gen, seqs, wl.lengths)
    cells = list(range(wl.n_cells))
    D, H = wl.head_dim, wl.n_heads
    qh = np.zeros((len(cells), len(seqs), H, g, D), np.uint16)
    for ci, c in enumerate(cells):
        for bl, b in enumerate(seqs):
            for h in range(H):
                qh[ci, bl, h] = W.query_group(wl, c, b, h, int(wl.lengths[b]), g)
    q = P.bits_to_bf16_tensor(qh, dev).contiguous()
    n = (len(cells), len(seqs), H)
    mw = int(wl.capacity.max()) // 32 + 1
    out = torch.empty(n + (g, D), dtype=torch.float32, device=dev)
    lse = torch.empty(n + (g,), dtype=torch.float32, device=dev)
    nsel = torch.empty(n, dtype=torch.int32, device=dev)
    mask = torch.zeros(n + (mw,), dtype=torch.int32, device=dev)
    plan.decode(cells, q, out=out, lse=lse, mask=mask, nsel=nsel)
    torch.cuda.synchronize()
    plan.check()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    nsel, mask = nsel.cpu().numpy(), mask.cpu().numpy().view(np.uint32)
    units = [(ci, bl, h) for ci in range(len(cells)) for bl in range(len(seqs)) for h in range(H)]
    jobs = [(spec, cells[ci], seqs[bl], h, int(wl.lengths[seqs[bl]]), int(wl.lengths[seqs[bl]]), g)
            for ci, bl, h in units]
    refs = pool.map(P.oracle_group_job, jobs)
    for (ci, bl, h), ref in zip(units, refs):
        tag = "g%d cell%d b%d h%d (%s)" % (g, cells[ci], seqs[bl], h, W.KIND_NAMES[ref["kind"]])
        assert (ref["q"] == qh[ci, bl, h]).all(), tag
        P.check_unit(tag, ref, out[ci, bl, h], lse=lse[ci, bl, h], mask=mask[ci, bl, h],
                     nsel=nsel[ci, bl, h], tau=wl.tau)
    return plan


@pytest.mark.parametrize("g", [2, 4])
@pytest.mark.parametrize("D", [64, 128])
def test_group_decode_matches_oracle(pool, cuda_device, g, D):
    lengths = (1, 33, 97, 300)
    for kinds in ((Q4, SH, Q2, Q4), (BF, SH, Q4, BF)):
        _run(_spec(D, kinds, lengths, 0.02), g, pool, cuda_device)


@pytest.mark.parametrize("g", [2, 4])
@pytest.mark.parametrize("D", [64, 128])
def test_group_residual_cells(pool, cuda_device, g, D):
    RS = W.RES2
    lengths = (1, 33, 97, 300)
    for kinds in ((RS, RS, Q4, Q2), (RS, SH, BF, Q4)):
        _run(_spec(D, kinds, lengths, 0.02), g, pool, cuda_device)


@pytest.mark.parametrize("g", [2, 4])
def test_group_residual_cells_in_clusters(pool, cuda_device, g):
    _run(_spec(128, (W.RES2, W.RES2, Q4, Q2), (65, 700, 1500), 0.01), g, pool, cuda_device,
         split=2)


@pytest.mark.parametrize("g", [2, 4])
@pytest.mark.parametrize("tau", [0.0, 2.0])
def test_group_tau_extremes(pool, cuda_device, tau, g):
    _run(_spec(128, (Q4, SH, Q2, Q4), (40, 300, 1000), tau), g, pool, cuda_device)


@pytest.mark.parametrize("g", [2, 4])
@pytest.mark.parametrize("split", [2, 4])
def test_group_cluster_split(pool, cuda_device, split, g):
    _run(_spec(128, (Q4, SH, Q2, Q4), (65, 700, 1500), 0.01), g, pool, cuda_device, split=split)


def test_group_long_units_split_automatically(pool, cuda_device):
    # four query heads leave fewer score slots per query in a CTA: long
    # units go to clusters without being asked
    _run(_spec(128, (Q4, SH, Q2, Q4), (9000,), 0.002, H=1), 4, pool, cuda_device)


@pytest.mark.parametrize("g", [2, 4])
def test_group_decode_16k_shape_sampled(pool, cuda_device, g):
    """The batched 16K workload's shape (16384 tokens per unit, 16 KV heads,
    head dim 128, its outlier keys and plan) with g query heads per KV head:
    8 cells covering every kind, 4 of its sequences, queries from the device
    generator, decoded in one launch per sort as the bench times it; sampled
    units against the oracle's group decode (every head's output and
    logsumexp, the KV head's union mask and count)."""
    import torch
    from loop_aware_quantized_b200 import Plan
    from synth.gpu import DeviceGenerator
    wl = W.make("2")
    seqs = [0, 9, 22, 31]
    # three Q4 (one in the final loop), three Q2, two SHARE cells
    cells = [0, 3, 13, 22, 30, 33, 35, 80]
    need = sorted(set(cells) | {wl.source_cell(c) for c in cells
                                if wl.kinds[c] in (SH, W.RES2)})
    plan = Plan(wl.n_loops, wl.n_layers, wl.n_heads, wl.head_dim, wl.capacity[seqs], wl.kinds,
                wl.tau, q_per_kv=g)
    gen = DeviceGenerator(wl, cuda_device)
    GH.build_cache(wl, plan, gen, seqs, wl.lengths[seqs], cells=need)
    lens = np.tile(wl.lengths[seqs], (len(cells), 1)).astype(np.int32)
    q = gen.queries(cells, seqs, lens, g=g)
    H, D = wl.n_heads, wl.head_dim
    n = (len(cells), len(seqs), H)
    mw = int(wl.capacity.max()) // 32 + 1
    out = torch.empty(n + (g, D), dtype=torch.float32, device=cuda_device)
    lse = torch.empty(n + (g,), dtype=torch.float32, device=cuda_device)
    nsel = torch.empty(n, dtype=torch.int32, device=cuda_device)
    mask = torch.zeros(n + (mw,), dtype=torch.int32, device=cuda_device)
    plan.decode(cells, q, out=out, lse=lse, mask=mask, nsel=nsel)
    torch.cuda.synchronize()
    plan.check()
    qh = q.view(torch.int16).cpu().numpy().view(np.uint16)
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    nsel, mask = nsel.cpu().numpy(), mask.cpu().numpy().view(np.uint32)
    units = GH.sample_units(wl, cells, seqs, 12, seed=50 + g)
    jobs = [("2", cells[ci], seqs[bl], h, int(wl.lengths[seqs[bl]]), int(wl.lengths[seqs[bl]]), g)
            for ci, bl, h in units]
    refs = pool.map(P.oracle_group_job, jobs)
    kinds = set()
    for (ci, bl, h), ref in zip(units, refs):
        tag = "16k g%d cell%d b%d h%d (%s)" % (g, cells[ci], seqs[bl], h,
                                              W.KIND_NAMES[ref["kind"]])
        assert (ref["q"] == qh[ci, bl, h]).all(), tag + ": device query differs from host"
        P.check_unit(tag, ref, out[ci, bl, h], lse=lse[ci, bl, h], mask=mask[ci, bl, h],
                     nsel=nsel[ci, bl, h], tau=wl.tau)
        kinds.add(ref["kind"])
    assert {Q4, Q2, SH} <= kinds
