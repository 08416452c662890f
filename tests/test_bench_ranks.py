"""The multi-rank reduction of bench.py on CPU: two gloo ranks."""
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t, us = bench.job_time(torch, dist, 1.0 + rank, steps=10, world=world, device="cpu")
        assert t == 2.0, t                        # the slowest rank's time
        assert abs(us - 2.0 / 20 * 1e6) < 1e-6    # all ranks' tokens over that time
    finally:
        dist.destroy_process_group()


def test_job_time_is_max_over_two_gloo_ranks():
    torch.multiprocessing.spawn(_rank, args=(2, _free_port()), nprocs=2, join=True)


def test_job_time_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    t, us = bench.job_time(torch, None, 0.5, steps=4, world=1, device="cpu")
    assert t == 0.5 and us == 0.5 / 4 * 1e6
