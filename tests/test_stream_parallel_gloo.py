"""The host side of stream parallelism with two ``gloo`` ranks on CPU: the
stream partition, the collective that gathers the ranks' shards (rank order,
shapes), and the process-group view a rank takes.  The kernels that consume
the gathered data are covered on the GPU by tests/test_gpu_stream_parallel.py."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from stream_sequence_attention_b200 import stream_parallel as sp


def test_local_streams():
    assert sp.local_streams(4, 2, 0) == [0, 2]
    assert sp.local_streams(4, 2, 1) == [1, 3]
    assert sp.local_streams(8, 4, 3) == [3, 7]
    assert sp.local_streams(4, 1, 0) == [0, 1, 2, 3]
    for bad in [(4, 3, 0), (4, 2, 2), (4, 0, 0)]:
        with pytest.raises(ValueError):
            sp.local_streams(*bad)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        n = 4
        view = sp.StreamParallel(n)
        assert (view.R, view.r, view.n_loc) == (world, rank, n // world)
        assert view.streams == list(range(rank, n, world))
        # Each rank's K shard holds its own streams: value = global stream id.
        B, L, H, D = 2, 3, 2, 4
        k_loc = torch.empty(B, L * view.n_loc, H, D)
        for i in range(L):
            for l, s in enumerate(view.streams):
                k_loc[:, i * view.n_loc + l] = s
        g = sp.all_gather_shards(k_loc)
        assert g.shape == (world, B, L * view.n_loc, H, D)
        for rr in range(world):
            for l, s in enumerate(sp.local_streams(n, world, rr)):
                assert torch.all(g[rr][:, l::view.n_loc] == s)
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, "ok"))
    except Exception as e:  # pragma: no cover - reported to the parent
        q.put((rank, repr(e)))


def test_two_rank_gather_of_stream_shards():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert res == {0: "ok", 1: "ok"}, res
