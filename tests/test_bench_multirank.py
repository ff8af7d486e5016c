"""The multi-rank host path of bench.py on CPU (gloo, world size 2): the
device time is the max over ranks, the value is whole-job throughput, and
only rank 0 runs the oracle reference arm."""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(10.0 + rank * 5.0, world, device="cpu")
        value = bench.weak_scaling_value(2e12, 10, world, ms)
        ref = bench.run_reference(type("A", (), {"workload": "tiny", "steps": 1, "warmup": 3})(), rank, world) \
            if rank == 1 else None
        out[rank] = (ms, value, ref)
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_value():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0          # the slowest rank's time
    expect = 2 * 2e12 * 10 / 15e-3 / 1e12
    assert abs(res[0][1] - expect) < 1e-9 and res[0][1] == res[1][1]
    assert res[1][2] is None                        # rank 1 skips the reference arm


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.weak_scaling_value(1e12, 4, 1, 2.0) == pytest.approx(2000.0)
