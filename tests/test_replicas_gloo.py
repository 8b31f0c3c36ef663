"""The multi-GPU path of bench.py runs independent replicas: each rank times
its own copy of the workload, the job time is the slowest rank's, and the
reported value is all ranks' bytes over that time.  This checks that host
logic with two gloo ranks on CPU (no GPU, no NCCL)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [2.0, 5.0][rank]  # rank 1 is the slow replica
        ms = bench.max_over_ranks(local_ms, world)
        v = bench.job_rate(1e6, 10, world, ms)
        q.put((rank, ms, v))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms, v in got:
        assert ms == 5.0  # both ranks agree on the slowest rank's time
        # 2 ranks x 10 steps x 1 MB in 5 ms
        assert v == pytest.approx(2 * 10 * 1e6 / 5e-3 / 1e9)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_rate(2e9, 1, 1, 1000.0) == pytest.approx(2.0)
