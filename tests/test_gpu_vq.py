"""LoopVQ decode and encoder on the CUDA path against the CPU oracle (needs a B200):
ragged lengths, every loop, both head dims, cluster splits, the device input
generator, the 16K shape on sampled units, the host argument checks, and
bit-exact nearest-entry indices from the encoder."""

import numpy as np
import pytest

from synth import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu


def _oracle_vq_job(args):
    """Oracle decode of one LoopVQ unit, inputs from the host generator."""
    from oracle import oracle as orc
    wl_args, loop, layer, b, h, n = args
    wl = W.make_vq(*wl_args[:1], **wl_args[1])
    ik = W.vq_indices(wl, 0, layer, b, h, 0, n)
    iv = W.vq_indices(wl, 1, layer, b, h, 0, n)
    cbk = W.vq_codebook(wl, 0, layer, h)
    cbv = W.vq_codebook(wl, 1, layer, h)
    q = W.vq_query(wl, loop, layer, b, h)
    out, lse = orc.vq_decode(ik, iv, cbk, cbv, q, loop, wl.n_loops)
    return dict(out=out, lse=lse, q=q)


@pytest.fixture(scope="module")
def pool():
    p = P.make_pool(8)
    yield p
    p.terminate()


def _run(wl_args, loops, pool, dev, units=None):
    import torch
    from loop_aware_quantized_b200 import vq_decode
    from synth.gpu import VqDeviceGenerator
    wl = W.make_vq(wl_args[0], **wl_args[1])
    gen = VqDeviceGenerator(wl, dev)
    ik, iv = gen.indices(0), gen.indices(1)
    cbk, cbv = gen.codebooks(0), gen.codebooks(1)
    if units is None:
        units = [(layer, b, h) for layer in range(wl.n_layers) for b in range(wl.batch)
                 for h in range(wl.n_heads)]
    for loop in loops:
        q = gen.queries(loop)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
        out = vq_decode(loop, wl.lengths, ik, iv, cbk, cbv, q, lse=lse)
        torch.cuda.synchronize()
        out, lse = out.cpu().numpy(), lse.cpu().numpy()
        qh = q.view(torch.int16).cpu().numpy().view(np.uint16)
        jobs = [(wl_args, loop, layer, b, h, int(wl.lengths[b])) for layer, b, h in units]
        for (layer, b, h), ref in zip(units, pool.map(_oracle_vq_job, jobs)):
            tag = "%s loop %d layer %d b %d h %d" % (wl.name, loop, layer, b, h)
            assert (qh[layer, b, h] == ref["q"]).all(), tag + ": device query differs from host"
            P.check_unit(tag, dict(out=ref["out"], lse=ref["lse"]),
                         out[layer, b, h], lse=lse[layer, b, h])


@pytest.mark.parametrize("D", [64, 128])
def test_vq_small_every_loop(pool, cuda_device, D):
    _run(("vqsmall", {"head_dim": D}), range(4), pool, cuda_device)


@pytest.mark.parametrize("n_loops", [1, 2, 8])
def test_vq_loop_counts(pool, cuda_device, n_loops):
    _run(("vqsmall", {"n_loops": n_loops}), [0, n_loops - 1], pool, cuda_device)


def test_vq_long_units_use_clusters(pool, cuda_device):
    # 20000 tokens need three CTAs' score slots: a cluster of four
    over = {"batch": 2, "lengths": np.array([20000, 9000], np.int32), "capacity": 20000,
            "n_layers": 1}
    _run(("vqsmall", over), [1], pool, cuda_device)


def test_vq_device_generator_matches_host(cuda_device):
    import torch
    from synth.gpu import VqDeviceGenerator
    wl = W.make_vq("vqsmall")
    gen = VqDeviceGenerator(wl, cuda_device)
    for which in (0, 1):
        d = gen.indices(which).cpu().numpy()
        for layer, b, h in ((0, 0, 0), (1, 2, 1)):
            assert (d[layer, b, h, :50] == W.vq_indices(wl, which, layer, b, h, 0, 50)).all()
    q = gen.queries(3).view(torch.int16).cpu().numpy().view(np.uint16)
    assert (q[1, 2, 1] == W.vq_query(wl, 3, 1, 2, 1)).all()
    # a rank's generator starts at its first global sequence
    g5 = VqDeviceGenerator(wl, cuda_device, seq0=5)
    d = g5.indices(1).cpu().numpy()
    assert (d[1, 2, 0, :40] == W.vq_indices(wl, 1, 1, 7, 0, 0, 40)).all()
    q = g5.queries(2).view(torch.int16).cpu().numpy().view(np.uint16)
    assert (q[0, 1, 1] == W.vq_query(wl, 2, 0, 6, 1)).all()


def test_vq_16k_shape_sampled(pool, cuda_device):
    # the benchmark's shape; oracle on a seeded sample of units
    rng = np.random.default_rng(3)
    units = [(int(rng.integers(24)), int(rng.integers(32)), int(rng.integers(16))) for _ in range(6)]
    _run(("vq16k", {}), [0, 3], pool, cuda_device, units=units)


def test_vq_argument_checks(cuda_device):
    import torch
    from loop_aware_quantized_b200 import LoopKVError, vq_decode
    wl = W.make_vq("vqsmall")
    ik = torch.zeros((2, 3, 2, 704, 32), dtype=torch.uint8, device=cuda_device)
    cb = torch.zeros((2, 2, 256, 16), dtype=torch.float32, device=cuda_device)
    q = torch.zeros((2, 3, 2, 128), dtype=torch.bfloat16, device=cuda_device)
    vq_decode(0, wl.lengths, ik, ik, cb, cb, q)
    for loop, lens in ((4, wl.lengths), (-1, wl.lengths), (0, np.array([0, 1, 1])),
                       (0, np.array([1, 1, 705]))):
        with pytest.raises(LoopKVError):
            vq_decode(loop, lens, ik, ik, cb, cb, q)
    torch.cuda.synchronize()


@pytest.mark.parametrize("D,L", [(128, 4), (64, 2), (128, 8)])
def test_vq_encode_matches_oracle(cuda_device, D, L):
    # nearest-entry indices, bit-exact: both sides compute the distances in
    # the same fp32 order and break ties to the lowest index
    import torch
    from loop_aware_quantized_b200 import vq_encode
    from oracle import oracle as orc
    from synth import philox as px
    wl = W.make_vq("vqsmall", head_dim=D, n_loops=L, batch=2, lengths=np.array([9, 9], np.int32),
                   capacity=16)
    n_new, pos = 5, np.array([3, 0], np.int32)
    shape = (L, wl.n_layers, wl.batch, wl.n_heads, n_new, D)
    u = px.philox4x32(np.arange(int(np.prod(shape)), dtype=np.uint32), 0, 0, 0, 77, 99)
    x = px.float_to_bf16_bits(px.normal_from_bits(*u).reshape(shape))
    cb = np.stack([np.stack([W.vq_codebook(wl, 0, layer, h) for h in range(wl.n_heads)])
                   for layer in range(wl.n_layers)])
    dx = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(cuda_device)
    dcb = torch.from_numpy(np.ascontiguousarray(cb)).to(cuda_device)
    idx = torch.zeros((wl.n_layers, wl.batch, wl.n_heads, 16, D // 4), dtype=torch.uint8,
                      device=cuda_device)
    vq_encode(pos, dx, dcb, idx)
    got = idx.cpu().numpy()
    for layer in range(wl.n_layers):
        for b in range(wl.batch):
            for h in range(wl.n_heads):
                for i in range(n_new):
                    want = orc.vq_encode(x[:, layer, b, h, i, :], cb[layer, h])
                    assert (got[layer, b, h, pos[b] + i] == want).all(), (layer, b, h, i)
                # positions outside the written range stay untouched
                untouched = [t for t in range(16) if not pos[b] <= t < pos[b] + n_new]
                assert (got[layer, b, h, untouched] == 0).all()


def test_vq_longest_unit_then_refusal(pool, cuda_device):
    # 8 CTAs of 8448 score slots hold 67584 tokens; one more is refused
    import torch
    from loop_aware_quantized_b200 import LoopKVError, vq_decode
    over = {"batch": 1, "lengths": np.array([67584], np.int32), "capacity": 67585, "n_layers": 1,
            "n_heads": 1}
    _run(("vqsmall", over), [2], pool, cuda_device)
    wl = W.make_vq("vqsmall", **over)
    ik = torch.zeros((1, 1, 1, 67585, 32), dtype=torch.uint8, device=cuda_device)
    cb = torch.zeros((1, 1, 256, 16), dtype=torch.float32, device=cuda_device)
    q = torch.zeros((1, 1, 1, 128), dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(LoopKVError) as e:
        vq_decode(0, np.array([67585], np.int32), ik, ik, cb, cb, q)
    assert e.value.status == 4
    torch.cuda.synchronize()
