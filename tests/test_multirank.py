"""The multi-GPU bench path (one process per GPU, replicas of the workload, step time = max
over ranks) exercised with two gloo ranks on the CPU: the cross-rank max, the whole-job
value and the reference arm's rank-0-only rule."""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench

    step_ms = [2.0, 3.5][rank]  # rank 1 is the slow one
    m = bench.reduce_max(step_ms, dist, "cpu")
    value = bench.job_value(4096, world, m)
    # the reference arm runs on rank 0 only; the other ranks return without work

    class Args:
        config, steps, warmup = "c1", 1, 1

    if rank != 0:
        bench.run_reference(Args, world, rank)
    out[rank] = (m, value)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_max_and_job_value():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        ps = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in ps:
            p.start()
        for p in ps:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0] == res[1]            # every rank sees the same aggregate
    m, value = res[0]
    assert m == pytest.approx(3.5)     # the slowest rank's step time
    assert value == pytest.approx(2 * 4096 / 3.5e-3)


def test_single_rank_helpers():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.reduce_max(1.25) == 1.25
    assert bench.job_value(64, 1, 2.0) == pytest.approx(32000.0)
