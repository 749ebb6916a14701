"""The multi-GPU bench path on CPU: world_size 2 with the gloo backend.

Every rank times its own share (weak scaling, no data-path collective); the
only cross-rank steps are the barrier and the max over ranks of the timed
region, which this test runs with gloo.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slower one
        dist.barrier()
        t = bench.max_over_ranks(torch, dist, local_ms, device="cpu")
        q.put((rank, t))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == {0: 15.0, 1: 15.0}


def test_seeds_differ_per_rank():
    # each rank draws its own batch (data-parallel): seeds are rank-dependent
    assert bench.rank_seed("intra", 0) != bench.rank_seed("intra", 1)
    assert bench.rank_seed("intra", 0) == bench.rank_seed("intra", 0)
