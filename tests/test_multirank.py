"""Host logic of the N-GPU benchmark on CPU ranks (gloo, world size 2): each
rank runs its own replica of the workload, the step time is the maximum over
ranks, and the job throughput counts every rank's units."""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = [3.0, 5.0][rank]                    # rank 1 is the slow one
        worst = bench.max_over_ranks(ms, world, device="cpu")
        q.put((rank, worst, bench.job_throughput(16640, worst, world)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, worst, value in res:
        assert worst == 5.0
        assert value == pytest.approx(2 * 16640 / 5e-3)


def test_single_rank_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.0, 1) == 4.0
    assert bench.job_throughput(100, 2.0, 1) == pytest.approx(5e4)
