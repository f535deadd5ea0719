"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

The decode path shards by (sequence, KV head) with no data exchange, so N GPUs run N
independent replicas; the only cross-rank steps are the timing reduction (max over ranks)
and the whole-job rate.  These run here as two gloo processes on 127.0.0.1.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist

    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 10.0 + 5.0 * rank              # rank 1 is the slow one
        m = bench.max_over_ranks(local_ms, torch.device("cpu"))
        rate = bench.whole_job_rate(world, 1000, m)
        # every rank takes part in the same collective steps, including a barrier
        dist.barrier()
        q.put((rank, m, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_rate_gloo_world2():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, m, rate in got:
        assert m == 15.0                           # the slowest rank's time on every rank
        assert rate == pytest.approx(2 * 1000 / 15e-3)


def test_single_process_rate_is_local():
    import torch

    import bench

    assert bench.max_over_ranks(7.5, torch.device("cpu")) == 7.5
    assert bench.whole_job_rate(1, 131072, 0.25) == pytest.approx(131072 / 0.25e-3)


def test_reference_arm_runs_on_rank0_only(monkeypatch):
    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = bench.main.__globals__["argparse"].Namespace(
        workload="single_head_T4096_R1", steps=1, warmup=0)
    assert bench.run_reference(args) is None
