"""The multi-rank path of bench.py on CPU: two gloo ranks shard sequences
without overlap and agree on the max-over-ranks timing.  The decode itself
needs no collective (units are independent)."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as tmp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        seqs = bench.shard_sequences(rank, 32)
        got = bench.max_over_ranks([10.0 + rank, 5.0 - rank], world, torch.device("cpu"))
        gathered = [None] * world
        dist.all_gather_object(gathered, seqs)
        out[rank] = (got, gathered)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_ranks_shard_and_reduce():
    world = 2
    mgr = tmp.Manager()
    out = mgr.dict()
    tmp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        got, gathered = out[r]
        assert got == [11.0, 5.0]
        flat = [s for g in gathered for s in g]
        assert len(flat) == len(set(flat)) == 64
