"""The N>1 plumbing of bench.py on CPU: two gloo ranks (world size 2).

The decode path shards by sequence (each GPU runs its own batch; no data-path
collective), so the multi-rank logic is the timing reduction (max over ranks),
the whole-job throughput and which rank reports.  These run the same helpers
bench.py uses under torchrun, over gloo on the host.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r is slower on a different quantity: the max must be taken element-wise
        mine = [10.0 + rank, 20.0 - rank, 5.0 + 2 * rank]
        dist.barrier()
        got = bench.max_over_ranks(mine, world)
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == out[1] == [11.0, 20.0, 7.0]


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.0, 2.0], 1) == [1.0, 2.0]


def test_job_throughput_is_whole_job():
    sys.path.insert(0, ROOT)
    import bench
    # 8 query tokens per step per rank, 20 steps in 100 ms on each of 4 ranks
    assert bench.job_throughput(4, 8, 20, 100.0) == pytest.approx(4 * 8 * 20 / 0.1)
    assert bench.job_throughput(1, 8, 20, 100.0) == pytest.approx(8 * 20 / 0.1)


def test_reference_arm_nonzero_rank_exits_without_work():
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W

    class A:
        steps, warmup = 3, 3
    # rank 1 of 2 returns at once (no oracle work, no output)
    assert bench.run_reference(A(), W.WORKLOADS["tiny"], rank=1, world=2) == 0
