"""The multi-GPU path of bench.py is one replica per rank with no data-path
exchange; its host logic (rendezvous, barrier, max-over-ranks timing, weak-
scaling aggregation) runs here as two gloo ranks on CPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime
    import sys

    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        dist.barrier()
        elapsed = 100.0 + 50.0 * rank  # rank 1 is the slow one
        worst = bench.max_over_ranks(elapsed, "cpu")
        ms, value, per_gpu = bench.aggregate(46_002_176, 1000, worst, world)
        out[rank] = (worst, ms, value, per_gpu)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_rank, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    assert out[0] == out[1]
    worst, ms, value, per_gpu = out[0]
    assert worst == 150.0
    assert ms == pytest.approx(0.15)
    assert per_gpu == pytest.approx(46_002_176 / 0.15e-3 / 1e9)
    assert value == pytest.approx(2 * per_gpu)


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    ms, value, per_gpu = bench.aggregate(1000, 10, 20.0, 1)
    assert ms == 2.0 and value == per_gpu
