"""RES2 cells (2-bit residuals against the final loop's KV) on the CUDA path
against the CPU oracle (needs a B200): cache bytes, outputs, masks and
counts over every reference kind, group and window boundaries, serving-order
appends, cluster splits, and the host checks on the reference."""

import numpy as np
import pytest

from synth import workloads as W
from tests import gpu_harness as GH
from tests.test_gpu_edges import _check_spec, _spec

pytestmark = pytest.mark.gpu

Q4, Q2, SH, BF, RS = W.Q4, W.Q2, W.SHARE, W.BF16, W.RES2


@pytest.fixture(scope="module")
def pool():
    from tests import parity as P
    p = P.make_pool(8)
    yield p
    p.terminate()


@pytest.mark.parametrize("D", [64, 128])
def test_residual_cells_match_oracle(pool, cuda_device, D):
    # window edges: 63 / 64 / 65 tokens move the residual-coded count 0 -> 32
    lengths = (1, 31, 63, 64, 65, 97, 200)
    for kinds in ((RS, RS, Q4, Q2), (RS, Q4, BF, Q4), (RS, SH, Q4, Q2)):
        _check_spec(_spec(D, kinds, lengths, 0.01), pool, cuda_device)


@pytest.mark.parametrize("tau", [0.0, 2.0])
def test_residual_tau_extremes(pool, cuda_device, tau):
    _check_spec(_spec(128, (RS, RS, Q4, Q2), (40, 300, 1000), tau), pool, cuda_device)


def test_residual_serving_order_appends(pool, cuda_device):
    # one token per step for every cell, loop-major: each residual group is
    # quantized one step after the reference holds it
    _check_spec(_spec(64, (RS, RS, Q4, BF), (1, 31, 64, 70, 130), 0.02), pool, cuda_device,
                token_by_token=True)


@pytest.mark.parametrize("split", [2, 4])
def test_residual_cluster_split(pool, cuda_device, split):
    _check_spec(_spec(128, (RS, Q2, Q4, Q4), (65, 700, 1500), 0.01), pool, cuda_device,
                split=split)


def test_residual_append_needs_its_reference(cuda_device):
    import torch
    from loop_aware_quantized_b200 import LoopKVError, Plan
    from synth.gpu import DeviceGenerator
    wl = W.custom(2, 1, 2, 64, (RS, Q4), (300,), (320,), 0.01)
    plan = Plan(2, 1, 2, 64, wl.capacity, wl.kinds, wl.tau)
    gen = DeviceGenerator(wl, cuda_device)

    def append(cell, t0, n):
        k, v = gen.kv([cell], [0], np.array([t0], np.int32), n)
        plan.append([cell], k, v)

    with pytest.raises(LoopKVError):
        append(0, 0, 100)           # the reference holds nothing yet
    assert plan.lengths()[0, 0] == 0
    append(0, 0, 63)                # nothing to quantize below 64 tokens
    append(1, 0, 100)               # reference: 96 quantized positions
    append(0, 63, 77)               # 140 tokens: 96 residual-coded
    with pytest.raises(LoopKVError):
        append(0, 140, 40)          # 180 tokens would need 160
    assert plan.lengths()[0, 0] == 140
    plan.check()
    torch.cuda.synchronize()


def test_residual_rollback_keeps_the_coded_range(pool, cuda_device):
    import torch
    from loop_aware_quantized_b200 import LoopKVError
    spec = _spec(64, (RS, RS, Q4, Q2), (130, 150), 0.02)
    plan = _check_spec(spec, pool, cuda_device)
    # 130 and 150 tokens: 96 residual-coded; 129 keeps 96, 127 would drop to 64
    with pytest.raises(LoopKVError):
        plan.set_lengths([0], np.array([[127, 150]], np.int32))
    plan.set_lengths([0], np.array([[129, 140]], np.int32))
    assert list(plan.lengths()[0, :2]) == [129, 140]
    torch.cuda.synchronize()


def test_residual_rollback_then_append(pool, cuda_device):
    """Window tokens dropped by set_lengths (or the whole unit reset) and
    appended again give the bytes and outputs of a fresh build."""
    import torch
    from synth.gpu import DeviceGenerator
    spec = _spec(64, (RS, Q2, Q4, Q4), (100, 150, 200), 0.02)
    wl = W.custom(*spec)
    seqs = [0, 1, 2]
    plan = GH.make_plan(wl, seqs)
    gen = DeviceGenerator(wl, cuda_device)
    cells = list(range(wl.n_cells))
    GH.build_cache(wl, plan, gen, seqs, wl.lengths)
    # residual-coded counts 64 / 96 / 160 stay; sequence 2 is reset
    back = np.array([97, 130, 0], np.int32)
    plan.set_lengths([0], back[None, :])
    assert (plan.lengths()[0, :3] == back).all()
    T = int((wl.lengths - back).max())
    k, v = gen.kv([0], seqs, back, T)
    plan.append([0], k, v, n_new=(wl.lengths - back).astype(np.int32))
    lens = np.tile(wl.lengths, (wl.n_cells, 1)).astype(np.int32)
    res = GH.decode_all(wl, plan, gen, seqs, cells, lens, cuda_device)
    plan.check()
    units = [(c, b, h) for c in cells for b in seqs for h in range(wl.n_heads)]
    n_of = lambda c, b: int(wl.lengths[b])  # noqa: E731
    GH.compare(spec, wl, plan, res, cells, seqs, units, n_of, n_of, pool)
    torch.cuda.synchronize()


def test_residual_reference_rounding_case(cuda_device):
    """The worked case where the reference's value needs two roundings,
    fl(fl(scale * code) + zero): a 4-bit reference key channel over
    [-2.71875, 2.953125] and a residual cell of zero keys, whose residual
    zero point is then -2.953125.  Both units' cache bytes equal the
    oracle's."""
    from loop_aware_quantized_b200 import Plan
    from oracle import oracle as orc
    from synth import philox as px
    from tests import parity as P
    D, n = 64, 64
    zeros = np.zeros((n, D), np.float32)
    kr = zeros.copy()
    kr[0, 0], kr[1, 0] = -2.71875, 2.953125
    bits = lambda a: px.float_to_bf16_bits(a)  # noqa: E731
    plan = Plan(2, 1, 1, D, np.array([128], np.int32), np.array([RS, Q4], np.uint8), 0.01,
                device=cuda_device)
    dev = lambda a: P.bits_to_bf16_tensor(bits(a)[None, None, None], cuda_device).contiguous()  # noqa: E731
    plan.append([1], dev(kr), dev(zeros))      # the final loop's cell: the reference
    plan.append([0], dev(zeros), dev(zeros))   # the residual cell
    ref = orc.OracleUnit(Q4, D, 128)
    ref.append(bits(kr), bits(zeros))
    own = orc.OracleUnit(RS, D, 128)
    own.append(bits(zeros), bits(zeros))
    assert own.export(src=ref)["kz"][0, 0] == np.float32(-2.953125)
    for cell, unit, src in ((1, ref, None), (0, own, ref)):
        want, valid = unit.serialize(src=src)
        P.check_bytes("reference rounding case, cell %d" % cell, dict(bytes=want, valid=valid),
                      plan.unit_bytes(cell, 0, 0).cpu().numpy())
    plan.check()
    plan.close()
