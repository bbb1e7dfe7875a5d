"""The benchmark's multi-rank host logic on CPU: two gloo ranks, as under torchrun.

The operator needs no exchange between GPUs (independent (batch, KV head) units), so
bench.py runs one replica per rank; the only collective is the max-over-ranks of the
device time, and the job value is the ranks' summed FLOPs over that slowest time.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    import bench
    ms_local = 10.0 + 5.0 * rank            # rank 1 is the slow one
    ms = bench.max_over_ranks(ms_local, world)
    value = bench.job_value(1.0e12, world, ms)
    out_q.put((rank, ms, value))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_max_time_and_job_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, value in got:
        assert ms == 15.0                    # every rank sees the slowest rank's time
        # 2 ranks x 1e12 FLOPs in 15 ms
        assert value == pytest.approx(2.0e12 / 15e-3 / 1e12)


def test_job_value_single_rank():
    import bench
    assert bench.job_value(2.0e12, 1, 20.0) == pytest.approx(100.0)
    assert bench.max_over_ranks(3.5, 1) == 3.5
