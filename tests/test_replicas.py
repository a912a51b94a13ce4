"""Multi-GPU replicas (world size 2) on the CPU: the bench's rank reduction takes the
slowest rank's time and counts every rank's units; every rank gets the same answer.
Runs two `gloo` ranks as processes (no GPU)."""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms_local = 10.0 + 5.0 * rank          # rank 1 is the slow one
        ms, value = bench.replica_throughput(ms_local, 1000.0, dist, "cpu")
        out[rank] = (ms, value)
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    import torch.multiprocessing as mp
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    for ms, value in res.values():
        assert ms == pytest.approx(15.0)                      # max over ranks
        assert value == pytest.approx(2 * 1000.0 / 0.015)     # both ranks' units / slowest time


def test_single_process_is_its_own_job():
    sys.path.insert(0, ROOT)
    import bench
    ms, value = bench.replica_throughput(8.0, 400.0)
    assert ms == 8.0 and value == pytest.approx(400.0 / 0.008)
