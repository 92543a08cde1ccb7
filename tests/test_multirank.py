"""The multi-GPU bench path on the CPU: two gloo ranks.

bench.py --gpus N runs one process per GPU, each compressing its own cache
(weak scaling, no collective on the data path).  The only cross-rank steps are
the barriers around the timed region and the max over ranks of the step time;
this test runs those helpers with world size 2 over gloo.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms, dist, torch.device("cpu"))
        value = bench.weak_scaling_value(1000, world, ms)
        dist.barrier()
        q.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_report_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, value in got:
        assert ms == 15.0                      # max over ranks, on every rank
        assert value == pytest.approx(2 * 1000 / 0.015)


def test_single_process_path_needs_no_group():
    import bench
    assert bench.max_over_ranks(3.5, None, torch.device("cpu")) == 3.5
    assert bench.weak_scaling_value(10, 1, 2.0) == pytest.approx(5000.0)
