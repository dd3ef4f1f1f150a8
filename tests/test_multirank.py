"""The benchmark's multi-rank host logic on two CPU ranks (gloo).

Every rank runs its own replica of the decode step; the only cross-rank
steps are the barriers around the timed region and the max of the ranks'
times.  These tests run those steps over a real two-process group."""
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        bench.barrier_if_distributed()
        ms = bench.max_over_ranks(times[rank], torch.device("cpu"))
        value = bench.whole_job_us_per_layer(ms, 32, world)
        bench.barrier_if_distributed()
        q.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value():
    world = 2
    times = [1.5, 4.0]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value in res:
        assert ms == max(times)                       # every rank sees the slowest rank
        assert value == pytest.approx(max(times) * 1e3 / (32 * world))


def test_whole_job_value_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5, torch.device("cpu")) == 2.5
    assert bench.whole_job_us_per_layer(1.0, 32, 1) == pytest.approx(1000.0 / 32)


def test_reference_arm_is_rank0_only(capsys):
    sys.path.insert(0, ROOT)
    import bench
    class A:
        workload, ref_layers, steps, warmup = 3, 8, 1, 0
    assert bench.run_reference(A(), rank=1, world=2) is None
    assert capsys.readouterr().out == ""


def test_selection_recall():
    """The bench's recall diagnostic: the share of the exact top-kappa (padding
    ignored) that a selection holds, per (batch, KV head) row."""
    sys.path.insert(0, ROOT)
    import bench
    sel = torch.tensor([[[0, 3, 5, -1], [1, 2, 3, 4]], [[-1, -1, -1, -1], [9, 10, 11, 12]]],
                       dtype=torch.int32)
    exact = torch.tensor([[[0, 5, 7, -1], [1, 2, 3, 4]], [[2, -1, -1, -1], [1, 2, 3, 4]]],
                         dtype=torch.int32)
    assert bench.selection_recall(sel, exact) == pytest.approx([2 / 3, 1.0, 0.0, 0.0])
    assert bench.selection_recall(exact, exact) == [1.0, 1.0, 1.0, 1.0]
