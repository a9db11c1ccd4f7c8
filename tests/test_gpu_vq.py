"""LoopVQ decode on the CUDA path against the CPU oracle (needs a B200):
ragged lengths, every loop, both head dims, cluster splits, the device input
generator, the 16K shape on sampled units, and the host argument checks."""

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
            P.check_unit(tag, dict(out=ref["out"], slack=np.zeros_like(ref["out"]), lse=ref["lse"]),
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
