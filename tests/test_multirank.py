"""The multi-rank bench logic on CPU (two gloo ranks): every rank reports the
slowest rank's time, and the whole-job value counts every rank's bytes over
that time. The path itself shards over batch and heads with no data-path
collective (replicas), so the timing reduction is the only exchange."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = 10.0 * (rank + 1)  # rank 1 is the slower one
        got = bench.max_over_ranks(ms, dist, torch.device("cpu"))
        out[rank] = (got, bench.whole_job_gbs(world, 1e9, 5, got))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 20.0
    # 2 ranks x 1 GB x 5 steps in 20 ms = 500 GB/s
    assert res[0][1] == pytest.approx(500.0) and res[1][1] == pytest.approx(500.0)


def test_single_process_passes_through():
    import bench
    assert bench.max_over_ranks(3.5, None, None) == 3.5
    assert bench.whole_job_gbs(1, 2e9, 10, 1000.0) == pytest.approx(20.0)
