"""Data-parallel path on CPU: two gloo ranks, each with its own batch of sequences.

The CSA2 decode path shards by sequence (every sequence has its own cache and indices), so ranks
exchange nothing on the data path; the only collective is the max of the step time over ranks.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = bench.rank_workload(workloads.TINY, rank)
        # a rank-specific workload draws its own data
        x = workloads.kv_chunk(wl, 0, 0, "cpu")
        digest = float(x.float().sum())
        ms = 10.0 + 5.0 * rank
        ms_max = bench.max_over_ranks(world, ms, torch.device("cpu"))
        value = bench.aggregate_value(world, wl.L, 4, ms_max)
        q.put((rank, wl.seed, digest, ms_max, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_by_sequence_and_take_max_time():
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
    (r0, s0, d0, m0, v0), (r1, s1, d1, m1, v1) = res
    assert s0 != s1 and d0 != d1          # independent batches
    assert m0 == m1 == 15.0               # both ranks report the slowest rank's time
    assert v0 == v1 == pytest.approx(2 * 1 * 4 / 0.015)  # whole-job layer-steps/s
