"""Multi-rank plumbing of bench.py on CPU (gloo, world_size 2): the elapsed
time is the max over ranks and the throughput counts every rank's steps."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    bench.init_dist("gloo", world)
    local_ms = 100.0 + 50.0 * rank          # rank 1 is the slowest
    max_ms = bench.reduce_max(local_ms, "cpu")
    bench.barrier("cpu")
    agg = bench.aggregate(world, flops_per_step=1e12, steps=10, max_ms=max_ms)
    q.put((rank, max_ms, agg))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_throughput():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, max_ms, agg in res:
        assert max_ms == 150.0
        # 2 ranks x 10 steps x 1e12 flop over 150 ms.
        assert agg["value"] == pytest.approx(2 * 10 * 1e12 / 0.150 / 1e12)
        assert agg["ms_per_step"] == pytest.approx(15.0)


def test_single_process_is_identity():
    import bench
    assert bench.reduce_max(3.5, "cpu") == 3.5
    agg = bench.aggregate(1, 2e12, 4, 8.0)
    assert agg["value"] == pytest.approx(4 * 2e12 / 0.008 / 1e12)


def test_step_flops_match_the_stated_counts():
    import bench
    from synth import WORKLOADS
    f = bench.step_flops(WORKLOADS["topk480"])
    assert f["sparse"] == pytest.approx(6.02e11, rel=2e-3)
    assert f["linear"] == pytest.approx(3.70e10, rel=2e-3)
    assert f["dense"] == pytest.approx(5.98e12, rel=2e-3)
    f4 = bench.step_flops(WORKLOADS["topk720"])
    assert f4["sparse"] == pytest.approx(2.09e13, rel=5e-3)
    assert bench.launches_per_step(WORKLOADS["topk480"]) == 8
