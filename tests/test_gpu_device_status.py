"""The device-side failure path on a B200, made on the host: one unit's length
in the device plan table is changed behind the host copy's back, so every
host check passes and the kernel alone can notice.  The kernel must flag it in
the table's status word, skip that unit (its outputs and cache bytes stay as
they were), and do everything else; loopkv_check then reports
LOOPKV_ERR_DEVICE once and clears the word.  Nothing here faults: both kernels
check the length before any access that depends on it."""

import numpy as np
import pytest

from synth import workloads as W
from tests import gpu_harness as GH

pytestmark = pytest.mark.gpu

Q4, Q2, SH = W.Q4, W.Q2, W.SHARE
SEQ_ENTRY = 32         # bytes per (cell, sequence) entry of the device table
LEN_FIELD = 20         # byte offset of the length inside an entry


def _len_offset(plan, cell, b):
    seqs = (256 + 16 * plan.n_cells + 255) // 256 * 256   # header, cells, 256-aligned
    return seqs + SEQ_ENTRY * (cell * plan.max_batch + b) + LEN_FIELD


def _poke_length(plan, cell, b, value):
    import torch
    off = _len_offset(plan, cell, b)
    old = plan.table[off:off + 4].clone()
    plan.table[off:off + 4] = torch.tensor([value], dtype=torch.int32).view(torch.uint8).to(
        plan.table.device)
    return old


def _device_length(plan, cell, b):
    import torch
    off = _len_offset(plan, cell, b)
    return int(plan.table[off:off + 4].cpu().view(torch.int32).item())


def _status_is_device_error(plan):
    from loop_aware_quantized_b200 import LoopKVError
    with pytest.raises(LoopKVError) as e:
        plan.check()
    assert e.value.status == 6       # LOOPKV_ERR_DEVICE
    plan.check()                     # reported once: the word is cleared


@pytest.fixture
def built(cuda_device):
    from synth.gpu import DeviceGenerator
    spec = (2, 2, 2, 64, (Q4, SH, Q2, Q4), (300, 200), (384, 256), 0.01)
    wl = W.custom(*spec)
    seqs = [0, 1]
    plan = GH.make_plan(wl, seqs)
    gen = DeviceGenerator(wl, cuda_device)
    GH.build_cache(wl, plan, gen, seqs, wl.lengths)
    plan.check()
    return wl, plan, gen, seqs


def test_table_length_offset_matches_the_host_copy(built):
    wl, plan, gen, seqs = built
    lens = plan.lengths()
    for c in range(wl.n_cells):
        for b in seqs:
            assert _device_length(plan, c, b) == lens[c, b]


@pytest.mark.parametrize("cell", [0, 1])          # a 4-bit unit; a SHARE unit
def test_decode_flags_a_unit_whose_device_length_is_zero(built, cuda_device, cell):
    import torch
    wl, plan, gen, seqs = built
    cells = list(range(wl.n_cells))
    lens = np.tile(wl.lengths, (wl.n_cells, 1)).astype(np.int32)
    good = GH.decode_all(wl, plan, gen, seqs, cells, lens, cuda_device)
    cache0 = plan.cache.clone()
    q = gen.queries(cells, seqs, lens)
    shape = (len(cells), len(seqs), wl.n_heads)
    out = torch.full(shape + (wl.head_dim,), float("nan"), device=cuda_device)
    lse = torch.full(shape, -7.0, device=cuda_device)
    nsel = torch.full(shape, -5, dtype=torch.int32, device=cuda_device)
    b = 1
    old = _poke_length(plan, cell, b, 0)               # the host copy still says 200
    plan.decode(cells, q, out=out, lse=lse, nsel=nsel)
    torch.cuda.synchronize()
    _status_is_device_error(plan)
    out, lse, nsel = out.cpu().numpy(), lse.cpu().numpy(), nsel.cpu().numpy()
    ci = cells.index(cell)
    assert np.isnan(out[ci, b]).all() and (lse[ci, b] == -7.0).all() and (nsel[ci, b] == -5).all()
    keep = np.ones(shape, bool)
    keep[ci, b] = False
    assert np.array_equal(out[keep], good["out"][keep])     # every other unit decoded as before
    assert np.array_equal(lse[keep], good["lse"][keep])
    assert torch.equal(plan.cache, cache0)
    plan.table[_len_offset(plan, cell, b):_len_offset(plan, cell, b) + 4] = old
    again = GH.decode_all(wl, plan, gen, seqs, cells, lens, cuda_device)
    plan.check()
    assert np.array_equal(again["out"], good["out"])


def test_append_flags_a_unit_whose_device_length_is_negative(built, cuda_device):
    import torch
    wl, plan, gen, seqs = built
    cells = list(range(wl.n_cells))
    cell, b = 0, 0
    before = [plan.unit_bytes(cell, b, h).clone() for h in range(wl.n_heads)]
    others = plan.unit_bytes(cell, 1, 0).clone()
    _poke_length(plan, cell, b, -1)                    # the host copy still says 300
    k, v = gen.kv(cells, seqs, wl.lengths.astype(np.int32), 1)
    plan.append(cells, k, v)
    torch.cuda.synchronize()
    _status_is_device_error(plan)
    for h in range(wl.n_heads):
        assert torch.equal(plan.unit_bytes(cell, b, h), before[h])   # nothing written
    assert not torch.equal(plan.unit_bytes(cell, 1, 0), others)      # the rest appended


def test_appends_commit_lengths_and_reset_their_arrival_counts(cuda_device):
    # the CTAs of a (cell, sequence) pair count their arrivals in the table;
    # the last one stores the new length and resets the count to zero.  A
    # bulk build of 1000 tokens spreads each unit over three CTAs.
    import torch
    from synth.gpu import DeviceGenerator
    spec = (2, 2, 2, 64, (Q4, SH, Q2, Q4), (1000, 600), (1120, 704), 0.01)
    wl = W.custom(*spec)
    seqs = [0, 1]
    plan = GH.make_plan(wl, seqs)
    gen = DeviceGenerator(wl, cuda_device)
    GH.build_cache(wl, plan, gen, seqs, wl.lengths)
    cells = list(range(wl.n_cells))
    lens = wl.lengths.astype(np.int32).copy()

    def check():
        torch.cuda.synchronize()
        plan.check()
        host = plan.lengths()
        for c in cells:
            for b in seqs:
                assert _device_length(plan, c, b) == host[c, b] == lens[b]
                off = _len_offset(plan, c, b) + 4
                assert int(plan.table[off:off + 4].cpu().view(torch.int32).item()) == 0

    check()
    for n_new in (1, 1, 5, 31, 60):            # token by token, a flush, a few groups
        k, v = gen.kv(cells, seqs, lens, n_new)
        plan.append(cells, k, v)
        lens += n_new
        check()
