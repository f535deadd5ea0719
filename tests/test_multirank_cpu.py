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


def test_kv_head_ranges_partition_every_head():
    import compressed_attention_cvq_b200 as cvq
    for n in (1, 2, 7, 8, 16):
        for world in (1, 2, 3, 4, 8):
            ranges = [cvq.kv_head_range(n, r, world) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [h1 - h0 for h0, h1 in ranges]
            assert max(sizes) - min(sizes) <= 1


def _shard_worker(rank, world, port, q):
    """Each rank decodes its KV heads of one small layer with the float64 oracle (the
    sharded inputs go through the same partition helper the benchmark uses); rank 0
    gathers the outputs."""
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist

    import workloads
    import compressed_attention_cvq_b200 as cvq
    from oracle import cvq_oracle as O

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        d = workloads.small(batch=2, n_q_heads=12, n_kv_heads=3, t_cap=96, R=2, seed=5,
                            seq_lens=np.array([96, 41], np.int32), cb_std=0.7071)
        shard, (h0, h1) = cvq.shard_kv_heads(d, 12, 3, rank, world)
        out, lse = O.attend(shard["q"], shard["key_cb"], shard["val_cb"], shard["key_codes"],
                            shard["val_codes"], shard["seq_lens"], d["rope_base"])
        # gather (out, lse) of every rank's query heads, padded to the largest shard
        g = 4
        pad_o = np.zeros((2, 2 * g, 128)); pad_l = np.zeros((2, 2 * g))
        pad_o[:, :out.shape[1]] = out; pad_l[:, :lse.shape[1]] = lse
        t = torch.from_numpy(np.concatenate([pad_o.ravel(), pad_l.ravel(), [h0, h1]]))
        parts = [torch.zeros_like(t) for _ in range(world)]
        dist.all_gather(parts, t)
        if rank == 0:
            ref_out, ref_lse = O.attend(d["q"], d["key_cb"], d["val_cb"], d["key_codes"],
                                        d["val_codes"], d["seq_lens"], d["rope_base"])
            n_o = 2 * 2 * g * 128
            for p in parts:
                p = p.numpy()
                a, b_ = int(p[-2]), int(p[-1])
                o = p[:n_o].reshape(2, 2 * g, 128)[:, :(b_ - a) * g]
                l = p[n_o:-2].reshape(2, 2 * g)[:, :(b_ - a) * g]
                assert np.array_equal(o, ref_out[:, a * g:b_ * g])
                assert np.array_equal(l, ref_lse[:, a * g:b_ * g])
        dist.barrier()
        q.put(rank)
    finally:
        dist.destroy_process_group()


def test_kv_head_partition_gloo_world2_equals_unsharded():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    assert sorted(q.get(timeout=10) for _ in range(world)) == [0, 1]
