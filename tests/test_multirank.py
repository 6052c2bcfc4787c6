"""The benchmark's multi-rank plumbing on CPU: two gloo ranks on 127.0.0.1.

Decode shards by sequence, so the ranks share no data-path collective; what
runs across ranks is the barrier around the timed region, the max over ranks
of its duration, and the reference arm, which rank 0 alone runs.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, out):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(ws), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import torch.distributed as dist
    got_ws, got_rank, _ = bench.dist_setup()
    bench.barrier(got_ws)
    # each rank's "timed region" differs; every rank must see the slowest
    slowest = bench.max_over_ranks(got_ws, 10.0 + 5.0 * got_rank)
    args = type("A", (), dict(workload=bench.DEFAULT_WORKLOAD, steps=1, warmup=3))()
    ref_line = bench.run_reference(args) if got_rank != 0 else "rank0-not-run"
    out.put((got_rank, got_ws, slowest, bench.shard_seed(got_rank, 0), bench.shard_seed(got_rank, 1),
             ref_line))
    bench.barrier(got_ws)
    dist.destroy_process_group()


def test_two_gloo_ranks_barrier_max_and_shards():
    ws, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, out)) for r in range(ws)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in range(ws)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert [r[0] for r in res] == [0, 1] and all(r[1] == ws for r in res)
    assert all(r[2] == 15.0 for r in res)  # the max over ranks, on every rank
    seeds = {s for r in res for s in (r[3], r[4])}
    assert len(seeds) == 4  # every (rank, layer) draws its own sequences
    assert res[1][5] is None  # rank 1 does no reference work


def test_job_throughput_counts_every_rank():
    # 16 sequences x 1 query per rank, 4 ranks, 10 steps in 20 ms (slowest rank)
    assert bench.job_throughput(16, 1, 4, 10, 20.0) == pytest.approx(16 * 4 * 10 / 0.020)
    assert bench.job_throughput(1, 4096, 1, 2, 10.0) == pytest.approx(4096 * 2 / 0.010)
