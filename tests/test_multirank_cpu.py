"""Host logic of the multi-GPU benchmark on two gloo ranks (CPU): the job time is the
slowest rank's time and the job throughput counts every rank's units."""
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


def _worker(rank, world, port, times, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = bench.max_over_ranks(times[rank], world, torch.device("cpu"))
        v = bench.job_throughput_gbs(1_000_000, 10, world, t)
        out[rank] = (t, v)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("times", [(3.0, 5.0), (7.5, 2.5)])
def test_max_over_ranks_gloo(times):
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, times, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    slowest = max(times)
    for r in range(2):
        t, v = out[r]
        assert t == slowest
        assert v == pytest.approx(1_000_000 * 10 * 2 / (slowest * 1e-3) / 1e9)


def test_single_rank_is_identity():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.max_over_ranks(4.0, 1, torch.device("cpu")) == 4.0
    assert bench.job_throughput_gbs(2e9, 1, 1, 1000.0) == pytest.approx(2.0)
