"""The multi-process path of bench.py on CPU with the gloo backend
(world_size 2): barrier, max of the per-rank times, one independent layer
per rank, whole-job aggregate.  No GPU and no data-path collective."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    from workloads import make_config
    ctx = bench.DistCtx()
    ctx.init("gloo")
    try:
        assert ctx.rank == rank and ctx.world == world
        ctx.barrier()
        # per-rank times: the job time is the slowest rank
        ms = 3.0 + rank
        ms_max = ctx.max(ms)
        # every rank runs its own layer: distinct seeded inputs
        wl = make_config(2, seqlen=256, seed=bench.rank_seed(rank))
        q_sum = float(wl.q.float().sum())
        sums = [ctx.max(q_sum if r == rank else -1e30) for r in range(world)]
        value = bench.weak_scaling_value(world, 1e12, ms_max)
        ctx.barrier()
        q.put((rank, ms_max, sums, value))
    finally:
        ctx.close()


def test_two_rank_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms_max, sums, value in res:
        assert ms_max == 3.0 + (world - 1)
        assert sums[0] != sums[1], "ranks must run independent (differently seeded) layers"
        # world x work / slowest rank: 2 x 1 TFLOP / 4 ms = 500 TFLOP/s
        assert value == pytest.approx(world * 1e12 / 4e-3 / 1e12)
    assert res[0][2] == res[1][2]
