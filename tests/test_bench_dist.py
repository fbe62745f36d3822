"""The benchmark's multi-process plumbing on the CPU (gloo, two ranks): each
rank runs its own workload (weak scaling, no collective on the data path),
the job's step time is the slowest rank's, and the whole-job throughput is
all ranks' flops over that time."""

import os
import socket
from datetime import timedelta

import pytest


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w, r, loc = bench.dist_setup(world)
        ms = bench.max_over_ranks(1.0 + rank, w, "cpu")  # rank 1 is the slower one
        q.put((r, w, loc, ms, bench.whole_job_tflops(3e12, w, ms)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_add_the_work():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    results.sort()
    assert [r[:3] for r in results] == [(0, 2, 0), (1, 2, 1)]
    for _, _, _, ms, value in results:
        assert ms == 2.0                     # the slowest rank's step, on every rank
        assert value == pytest.approx(3000.0)  # 2 x 3e12 flops in 2 ms


def test_single_process_rejects_more_than_one_gpu(monkeypatch):
    import bench

    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_setup(1) == (1, 0, 0)
    with pytest.raises(SystemExit):
        bench.dist_setup(2)
    assert bench.max_over_ranks(4.5, 1, "cpu") == 4.5
    assert bench.whole_job_tflops(1e12, 1, 1.0) == pytest.approx(1000.0)
