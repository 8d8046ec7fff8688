"""The N-GPU host logic of bench.py on CPU: two gloo ranks, each with its own
per-rank time, agree on the max (the slowest rank sets the step time) and on
the weak-scaling whole-job value."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t = bench.reduce_max(times[rank], dist, torch.device("cpu"), world)
        v = bench.whole_job_tflops(world, 1e12, t)
        out[rank] = (t, v)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_max_and_weak_scaling_value():
    world = 2
    times = [1.5, 2.0]
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    port = _free_port()
    mp.start_processes(_rank, args=(world, port, times, out), nprocs=world, join=True, start_method="spawn")
    assert out[0] == out[1]
    t, v = out[0]
    assert t == 2.0
    assert v == pytest.approx(world * 1e12 / 2e-3 / 1e12)
