"""The benchmark's multi-rank host logic on world_size 2 over gloo (CPU): each rank runs an
independent replica (distinct seeded batch), and timings are reduced as a max over ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime

    import bench
    import moe_inputs
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = moe_inputs.small(T=4, d=64, F=64)
        wr = bench.replica_workload(w, rank)
        x = moe_inputs.make_x(wr)
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 3.5])
        gathered = [None] * world
        dist.all_gather_object(gathered, x.float().sum().item())
        q.put((rank, got, gathered, bench._dist()))
    finally:
        dist.destroy_process_group()


def test_replicas_and_max_over_ranks_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, gathered, envdist in res:
        assert got == [2.0, 10.0, 3.5]                    # max over ranks, element-wise
        assert gathered[0] != gathered[1]                 # replicas draw different batches
        assert envdist == (world, rank, 0)                # RANK / WORLD_SIZE from the env


def test_single_rank_max_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
