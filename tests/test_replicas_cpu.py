"""The multi-GPU bench path on CPU: world size 2 over gloo. Every rank runs its own replica;
the timed region is the slowest rank's, and the value is the whole job's units over it."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        secs = [0.5, 2.0][rank]                      # rank 1 is the slow one
        slowest = bench.max_over_ranks_of(dist, secs)
        dist.barrier()
        out.put((rank, slowest, bench.replica_value(world, 100.0, slowest)))
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [2.0, 2.0]
    assert all(r[2] == pytest.approx(100.0) for r in res)     # 2 ranks x 100 units / 2.0 s


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks_of(None, 1.25) == 1.25
    assert bench.replica_value(1, 10.0, 2.0) == 5.0
