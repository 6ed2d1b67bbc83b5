"""The N>1 host path of bench.py on CPU: two gloo ranks, no GPU.

Each rank must get its own sequence (same shape, different seed), the timing
reduction must return the slowest rank's time on every rank, and the whole-job
rate must count all ranks' tokens over that time.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime

    import torch.distributed as dist

    import bench
    import workloads
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        w_world, w_rank, _ = bench.dist_env()
        assert (w_world, w_rank) == (world, rank)
        w = bench.rank_workload(workloads.WORKLOADS["gqa128k"], rank)
        my_ms = 10.0 + 5.0 * rank
        bench.barrier(world)
        slowest = bench.max_over_ranks(my_ms, world)
        rate = bench.whole_job_tokens_per_s(w.batch * w.seq_q, world, slowest)
        out.put((rank, w.seed, w.seq_q, slowest, rate))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reduce():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    seeds = {r[1] for r in res}
    assert len(seeds) == world                       # each rank its own sequence
    assert {r[2] for r in res} == {131072}            # same shape everywhere
    assert all(r[3] == 15.0 for r in res)             # slowest rank's time on every rank
    assert all(r[4] == pytest.approx(131072 * 2 / 0.015) for r in res)
