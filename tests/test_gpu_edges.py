"""Edge cases of the CUDA path against the CPU oracle (needs a B200): group
boundaries, one-token units, SHARE over partial groups and residuals,
token-by-token vs bulk append, rollback, tau extremes, argument errors."""

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


def _spec(D, kinds, lengths, tau, n_loops=2, n_layers=2, H=2, extra=64):
    cap = tuple(int((n + extra + 31) // 32 * 32) for n in lengths)
    return (n_loops, n_layers, H, D, tuple(kinds), tuple(lengths), cap, tau)


def _check_spec(spec, pool, dev, token_by_token=False, src_lengths=None, split=0):
    """Build all cells of a custom workload, decode every unit, oracle-check all
    (split: CTAs per decoded unit at least; 0 lets the library choose)."""
    import torch
    from synth.gpu import DeviceGenerator
    wl = W.custom(*spec)
    seqs = list(range(wl.batch))
    plan = GH.make_plan(wl, seqs, decode_split=split)
    gen = DeviceGenerator(wl, dev)
    cells = list(range(wl.n_cells))
    if token_by_token:
        T = int(wl.lengths.max())
        for t in range(T):
            n_new = (wl.lengths > t).astype(np.int32)
            k, v = gen.kv(cells, seqs, np.full(len(seqs), t, np.int32), 1)
            plan.append(cells, k, v, n_new=n_new)
    else:
        GH.build_cache(wl, plan, gen, seqs, wl.lengths)
    lens = np.tile(wl.lengths, (wl.n_cells, 1)).astype(np.int32)
    res = GH.decode_all(wl, plan, gen, seqs, cells, lens, dev)
    plan.check()
    units = [(c, b, h) for c in cells for b in seqs for h in range(wl.n_heads)]
    n_of = lambda c, b: int(wl.lengths[b])  # noqa: E731
    GH.compare(spec, wl, plan, res, cells, seqs, units, n_of, n_of, pool)
    torch.cuda.synchronize()
    return plan


@pytest.mark.parametrize("D", [64, 128])
def test_group_boundaries(pool, cuda_device, D):
    # lengths around group edges; SHARE sources of the same length
    lengths = (1, 2, 31, 32, 33, 63, 64, 65, 97)
    for kinds in ((Q4, SH, Q2, Q4), (Q2, SH, Q4, Q2), (BF, SH, Q4, BF), (Q4, Q2, BF, Q4)):
        _check_spec(_spec(D, kinds, lengths, 0.01), pool, cuda_device)


@pytest.mark.parametrize("tau", [0.0, 0.03, 2.0])
def test_tau_extremes(pool, cuda_device, tau):
    _check_spec(_spec(128, (Q4, SH, Q2, Q4), (40, 300, 1000), tau), pool, cuda_device)


def test_token_by_token_append_matches_oracle(pool, cuda_device):
    _check_spec(_spec(64, (Q4, SH, Q2, Q4), (1, 31, 32, 70), 0.02), pool, cuda_device,
                token_by_token=True)


def test_share_with_longer_source(pool, cuda_device):
    """SHARE unit shorter than its source: reads [0, n-1) of the source only,
    across the source's quantized groups and residual."""
    import torch
    from synth.gpu import DeviceGenerator
    spec = _spec(128, (SH, SH, Q4, Q2), (50, 70, 129), 0.01)
    wl = W.custom(*spec)
    seqs = [0, 1, 2]
    plan = GH.make_plan(wl, seqs)
    gen = DeviceGenerator(wl, cuda_device)
    src_extra = np.array([7, 30, 40], np.int32)   # the final loop is ahead
    GH.build_cache(wl, plan, gen, seqs, wl.lengths, cells=[0, 1])
    GH.build_cache(wl, plan, gen, seqs, wl.lengths + src_extra, cells=[2, 3])
    cells = [0, 1]
    lens = np.tile(wl.lengths, (2, 1)).astype(np.int32)
    res = GH.decode_all(wl, plan, gen, seqs, cells, lens, cuda_device)
    plan.check()
    units = [(ci, b, h) for ci in range(2) for b in seqs for h in range(wl.n_heads)]
    own = lambda c, b: int(wl.lengths[b])  # noqa: E731
    src = lambda c, b: int(wl.lengths[b] + src_extra[b])  # noqa: E731
    GH.compare(spec, wl, plan, res, cells, seqs, units, own, src, pool)
    torch.cuda.synchronize()


def test_rollback_then_append(pool, cuda_device):
    """set_lengths drops residual tokens or whole groups; appending again
    rewrites those positions and the state equals a fresh build."""
    from synth.gpu import DeviceGenerator
    spec = _spec(64, (Q4, Q2, Q2, Q4), (45, 96, 70), 0.02)
    wl = W.custom(*spec)
    seqs = [0, 1, 2]
    plan = GH.make_plan(wl, seqs)
    gen = DeviceGenerator(wl, cuda_device)
    cells = list(range(wl.n_cells))
    GH.build_cache(wl, plan, gen, seqs, wl.lengths)
    # roll back: seq0 into its residual (45 -> 40), seq1 by two groups (96 -> 32),
    # seq2 to 0 (reset)
    back = np.array([40, 32, 0], np.int32)
    plan.set_lengths(cells, np.tile(back, (len(cells), 1)))
    assert (plan.lengths()[:, :3] == back).all()
    # re-append the same tokens
    T = int((wl.lengths - back).max())
    k, v = gen.kv([0], seqs, back, T)
    for c in cells:
        kk, vv = gen.kv([c], seqs, back, T)
        plan.append([c], kk, vv, n_new=(wl.lengths - back).astype(np.int32))
    lens = np.tile(wl.lengths, (wl.n_cells, 1)).astype(np.int32)
    res = GH.decode_all(wl, plan, gen, seqs, cells, lens, cuda_device)
    plan.check()
    units = [(c, b, h) for c in cells for b in seqs for h in range(wl.n_heads)]
    n_of = lambda c, b: int(wl.lengths[b])  # noqa: E731
    GH.compare(spec, wl, plan, res, cells, seqs, units, n_of, n_of, pool)


def test_argument_errors(cuda_device):
    import torch
    from loop_aware_quantized_b200 import LoopKVError
    from synth.gpu import DeviceGenerator
    spec = _spec(64, (Q4, SH, Q2, Q4), (40, 40), 0.01, extra=0)
    wl = W.custom(*spec)
    plan = GH.make_plan(wl, [0, 1])
    gen = DeviceGenerator(wl, cuda_device)
    k, v = gen.kv([0], [0, 1], np.zeros(2, np.int32), 40)
    plan.append([0], k, v)
    # capacity: 40 + 40 > 64
    with pytest.raises(LoopKVError) as e:
        plan.append([0], k, v)
    assert e.value.status == 3
    assert (plan.lengths()[0, :2] == 40).all()
    # duplicate / out-of-range cells
    with pytest.raises(LoopKVError):
        plan.append([0, 0], torch.cat([k, k]), torch.cat([v, v]))
    with pytest.raises(LoopKVError):
        plan.decode([7], torch.zeros((1, 2, 2, 64), dtype=torch.bfloat16, device=cuda_device))
    # decoding an empty unit is rejected
    with pytest.raises(LoopKVError):
        plan.decode([2], torch.zeros((1, 2, 2, 64), dtype=torch.bfloat16, device=cuda_device))
    # SHARE unit longer than its source + 1 is rejected (cell 3 is empty)
    plan.append([1], k, v)
    with pytest.raises(LoopKVError):
        plan.decode([1], torch.zeros((1, 2, 2, 64), dtype=torch.bfloat16, device=cuda_device))
    # rollback rules: SHARE cannot be shortened
    with pytest.raises(LoopKVError):
        plan.set_lengths([1], np.array([[39, 40]], np.int32))
    # empty append is a no-op
    plan.append([0], k, v, n_new=np.zeros(2, np.int32))
    assert (plan.lengths()[0, :2] == 40).all()
    plan.check()


def test_planner_plan_drives_the_cache(pool, cuda_device):
    # a plan chosen by loopkv_plan_optimize (host) is loaded, filled and
    # decoded like any other, unit by unit against the oracle
    from loop_aware_quantized_b200 import plan_optimize
    damage = np.array([[1, 5, 3], [2, 6, 4], [0, 3, 9], [1, 2, 9]])
    kinds, cost = plan_optimize(2, 2, 64, damage, 9, 14 * 16, 0.0)
    assert sorted(set(int(k) for k in kinds)) == [Q4, Q2, SH], kinds
    _check_spec(_spec(64, tuple(int(k) for k in kinds), (33, 97, 300), 0.02), pool, cuda_device)


def test_longest_unit_then_refusal(pool, cuda_device):
    """The longest unit a decode takes (8 CTAs of 24576 score slots: a
    cluster of 8) matches the oracle; one past what 8 CTAs hold is refused
    on the host with LOOPKV_ERR_UNSUPPORTED."""
    import torch
    from loop_aware_quantized_b200 import LoopKVError
    spec = (1, 1, 1, 128, (Q4,), (196000,), (196032,), 0.002)
    _check_spec(spec, pool, cuda_device)
    from synth.gpu import DeviceGenerator
    wl = W.custom(1, 1, 1, 128, (Q4,), (196700,), (196736,), 0.002)
    plan = GH.make_plan(wl, [0])
    GH.build_cache(wl, plan, DeviceGenerator(wl, cuda_device), [0], wl.lengths)
    with pytest.raises(LoopKVError) as e:
        plan.decode([0], torch.zeros((1, 1, 1, 128), dtype=torch.bfloat16, device=cuda_device))
    assert e.value.status == 4
    torch.cuda.synchronize()


def test_decode_replays_from_a_cuda_graph(cuda_device):
    """loopkv_decode only enqueues work (no host synchronisation), so a
    decode captured into a CUDA graph replays with the eager results, bit
    for bit (the kernel's reductions have a fixed order)."""
    import torch
    from synth.gpu import DeviceGenerator
    spec = _spec(128, (Q4, SH, Q2, Q4), (300, 1000), 0.01)
    wl = W.custom(*spec)
    seqs = [0, 1]
    plan = GH.make_plan(wl, seqs)
    gen = DeviceGenerator(wl, cuda_device)
    GH.build_cache(wl, plan, gen, seqs, wl.lengths)
    cells = list(range(wl.n_cells))
    q = gen.queries(cells, seqs, np.tile(wl.lengths, (len(cells), 1)))
    eager = plan.decode(cells, q).clone()
    out = torch.zeros_like(eager)
    s = torch.cuda.Stream(device=cuda_device)
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        plan.decode(cells, q, out=out, stream=s)
    for _ in range(2):
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager)
    plan.check()


def test_serving_steps_replay_from_a_cuda_graph(cuda_device):
    """A whole serving sequence (three steps of append + decode for the
    non-final loops, then for the final loop) captured as one CUDA graph and
    replayed once gives the eager run's outputs, masks, counts and cache
    bytes, bit for bit: the calls only enqueue kernels, and the appends read
    and advance the lengths on the device.  The lengths start one token
    short of a group boundary (31 and 319), so the first captured append
    quantizes a group."""
    import torch
    from loop_aware_quantized_b200 import steps
    from synth.gpu import DeviceGenerator
    spec = _spec(128, (Q4, SH, Q2, Q4), (31, 319), 0.01)
    wl = W.custom(*spec)
    seqs = [0, 1]
    n0 = wl.lengths.astype(np.int32)
    phase = steps.phases(wl.n_loops, wl.n_layers)
    H, D, B = wl.n_heads, wl.head_dim, len(seqs)
    n_steps = 3
    gen = DeviceGenerator(wl, cuda_device)
    plans = [GH.make_plan(wl, seqs) for _ in range(2)]
    for plan in plans:
        plan.cache.zero_()  # bytes the layout leaves undefined start equal too
        GH.build_cache(wl, plan, gen, seqs, n0)
    # every step's inputs, shared by both runs
    ins = []
    for s in range(n_steps):
        qs, ks, vs = [], [], []
        for cells in phase:
            k, v = gen.kv(list(cells), seqs, n0 + s, 1)
            ks.append(k)
            vs.append(v)
            qs.append(gen.queries(list(cells), seqs, np.tile(n0 + s + 1, (len(cells), 1))))
        ins.append((qs, ks, vs))
    mw = int(wl.capacity.max()) // 32 + 1

    def outputs():
        res = []
        for _ in range(n_steps):
            shp = [(len(c), B, H) for c in phase]
            res.append(dict(out=[torch.zeros(x + (D,), dtype=torch.float32, device=cuda_device)
                                 for x in shp],
                            lse=[torch.zeros(x, dtype=torch.float32, device=cuda_device)
                                 for x in shp],
                            mask=[torch.zeros(x + (mw,), dtype=torch.int32, device=cuda_device)
                                  for x in shp],
                            nsel=[torch.zeros(x, dtype=torch.int32, device=cuda_device)
                                  for x in shp]))
        return res

    def run(plan, res, stream=None):
        for s in range(n_steps):
            qs, ks, vs = ins[s]
            r = res[s]
            steps.decode_step(plan, phase, qs, ks, vs, r["out"], lse=r["lse"], mask=r["mask"],
                              nsel=r["nsel"], stream=stream)

    eager = outputs()
    run(plans[0], eager)
    torch.cuda.synchronize()
    replay = outputs()
    s = torch.cuda.Stream(device=cuda_device)
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        run(plans[1], replay, stream=s)
    # nothing ran during the capture: the cache still holds the bulk build
    torch.cuda.synchronize()
    assert not torch.equal(plans[1].cache, plans[0].cache)
    graph.replay()
    torch.cuda.synchronize()
    for s_ in range(n_steps):
        for key in ("out", "lse", "mask", "nsel"):
            for i in range(len(phase)):
                assert torch.equal(eager[s_][key][i], replay[s_][key][i]), (s_, key, i)
    assert torch.equal(plans[0].cache, plans[1].cache)
    for plan in plans:
        plan.check()
        assert (plan.lengths()[:, :B] == n0 + n_steps).all()
    del graph


def test_kernels_write_only_the_layout_bytes(pool, cuda_device):
    """Guard check (stands in for a memory checker): the cache is filled with
    a sentinel before a bulk build of every kind; afterwards every byte the
    canonical layout does not define at the units' lengths still holds the
    sentinel, and so do the guard bytes after the cache."""
    import torch
    from loop_aware_quantized_b200 import Plan
    from synth.gpu import DeviceGenerator
    RS = W.RES2
    spec = _spec(64, (RS, SH, Q4, Q2, BF, Q4), (45, 96, 70), 0.02, n_loops=2, n_layers=3)
    wl = W.custom(*spec)
    seqs = [0, 1, 2]
    guard = 1 << 16
    plan = Plan(wl.n_loops, wl.n_layers, wl.n_heads, wl.head_dim, wl.capacity[seqs], wl.kinds,
                wl.tau, cache_guard=guard)
    plan.cache.fill_(0xA5)
    gen = DeviceGenerator(wl, cuda_device)
    GH.build_cache(wl, plan, gen, seqs, wl.lengths)
    cells = list(range(wl.n_cells))
    GH.decode_all(wl, plan, gen, seqs, cells, np.tile(wl.lengths, (wl.n_cells, 1)), cuda_device)
    plan.check()
    torch.cuda.synchronize()
    assert (plan.cache[plan.cache_bytes:].cpu().numpy() == 0xA5).all(), "write past the cache"
    jobs = [(spec, c, b, h, int(wl.lengths[b]), int(wl.lengths[b]), True)
            for c in cells for b in seqs for h in range(wl.n_heads)]
    for (c, b, h), ref in zip([(j[1], j[2], j[3]) for j in jobs], pool.map(P.oracle_unit_job, jobs)):
        got = plan.unit_bytes(c, b, h).cpu().numpy()
        outside = ref["valid"] == 0
        bad = np.nonzero(outside & (got != 0xA5))[0]
        assert bad.size == 0, "cell %d seq %d head %d: %d stray bytes, first at %d" % (
            c, b, h, bad.size, bad[0])


def _division_case_tokens(D, hi, mid):
    """32 tokens whose every key channel and every value group is {0, hi,
    mid, 0, ...}: keys quantize per channel over the tokens, values per token
    over 32-channel groups.  hi and mid are exact in bf16."""
    k = np.zeros((32, D), np.float32)
    k[1, :], k[2, :] = hi, mid
    v = np.zeros((32, D), np.float32)
    for j in range(0, D, 32):
        v[:, j + 1], v[:, j + 2] = hi, mid
    bits = lambda a: (a.view(np.uint32) >> 16).astype(np.uint16)  # noqa: E731  exact here
    return bits(k), bits(v)


@pytest.mark.parametrize("D", [64, 128])
def test_quantizer_division_cases(cuda_device, D):
    """Groups whose codes hang on the fp32 ratio being one correctly rounded
    division (4 bits: scale fl32(1.125 / 15), 0.5625 -> code 7; 2 bits: scale
    fl32(1.625 / 3), 0.8125 -> code 2; a multiply by the scale's rounded
    reciprocal gives 8 and 1): the appended cache bytes equal the oracle's."""
    from loop_aware_quantized_b200 import Plan
    from oracle import oracle as orc
    for kind, hi, mid in ((Q4, 1.125, 0.5625), (Q2, 1.625, 0.8125)):
        kb, vb = _division_case_tokens(D, hi, mid)
        plan = Plan(1, 1, 1, D, np.array([64], np.int32), np.array([kind], np.uint8), 0.01,
                    device=cuda_device)
        plan.append([0], P.bits_to_bf16_tensor(kb[None, None, None], cuda_device).contiguous(),
                    P.bits_to_bf16_tensor(vb[None, None, None], cuda_device).contiguous())
        got = plan.unit_bytes(0, 0, 0).cpu().numpy()
        unit = orc.OracleUnit(kind, D, 64)
        unit.append(kb, vb)
        ref_bytes, valid = unit.serialize()
        P.check_bytes("division case kind %d D %d" % (kind, D), dict(bytes=ref_bytes, valid=valid),
                      got)
        plan.check()
        plan.close()
