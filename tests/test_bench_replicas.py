"""The multi-GPU path of bench.py is replicas only: each rank generates its own batch and the
ranks exchange nothing but the max of their timings.  Checked here with two gloo ranks on CPU."""
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


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms, wall = [1000.0 + 250.0 * rank], [2.0 - rank]
        got = bench.reduce_over_ranks(ms + wall, world, "cpu")
        tps = bench.whole_job_tokens_per_s(1, 256, 3, world, got[0] / 1e3)
        q.put((rank, got, tps))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_reduction_and_whole_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, tps in res:
        assert got == [1250.0, 2.0]                  # the slowest rank decides both clocks
        assert tps == pytest.approx(2 * 256 * 3 / 1.25)


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_over_ranks([3.5, 7.0], 1) == [3.5, 7.0]
