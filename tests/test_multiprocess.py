"""The multi-GPU bench path on CPU: world size 2 over gloo.  Each rank works on
its own batch (no data-path collective); timings are reduced with a max over
ranks and only rank 0 reports.  No GPU needed."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, lr, ws = bench.dist_env()
        assert (r, lr, ws) == (rank, rank, world)
        # every rank times its own work; the slowest rank sets the job's time
        mine = [10.0 + rank, 50.0 - rank, 8.0 + 2 * rank]
        total_ms, e2e_ms, fine_ms = bench.max_over_ranks(mine)
        agg = bench.aggregate(ws, 1e12, 10, total_ms, e2e_ms, fine_ms)
        results[rank] = (total_ms, e2e_ms, fine_ms, agg["value"], bench.rank_seed(2, rank))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_distinct_batches():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    r0, r1 = results[0], results[1]
    assert r0[:3] == r1[:3] == (11.0, 50.0, 10.0)            # max over ranks, everywhere
    # two ranks each did 1e12 FLOP per step in 11 ms / 10 steps = 1.1 ms per step
    assert r0[3] == pytest.approx(2 * 1e12 / 1.1e-3 / 1e12)
    assert r0[4] != r1[4]                                      # different input batches


def test_single_process_aggregate_is_identity():
    assert bench.max_over_ranks([1.0, 2.0]) == [1.0, 2.0]
    agg = bench.aggregate(1, 2e12, 4, 8.0, 10.0, 6.0)
    assert agg["ms_per_step"] == 2.0 and agg["value"] == pytest.approx(1000.0)
    assert agg["fine_ms"] == 1.5
