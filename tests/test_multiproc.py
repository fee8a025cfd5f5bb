"""The N > 1 host logic of bench.py on two CPU ranks (gloo): every rank runs
an independent call, the job time is the slowest rank's, and the job's ms per
call is that time divided by the calls all ranks made."""
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


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.argv = ["bench.py"]
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_step_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        bench.barrier(world)
        out[rank] = (bench.max_over_ranks(local_step_ms, world), bench.job_ms_per_call(local_step_ms, world))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_and_weak_scaling():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    for r in range(world):
        slowest, per_call = res[r]
        assert slowest == pytest.approx(15.0)
        assert per_call == pytest.approx(7.5)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    sys.argv = ["bench.py"]
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25
    assert bench.job_ms_per_call(3.25, 1) == 3.25
