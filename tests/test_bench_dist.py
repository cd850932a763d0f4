"""The bench's multi-process plumbing on the CPU: two gloo ranks (no GPU).  Several GPUs run independent
replicas of the step, so the only traffic between ranks is the timing scalars: the whole-job value is the
bytes all ranks moved over the slowest rank's time, and every rank takes the same collective steps."""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        bench.barrier(world)
        ms = 10.0 * (rank + 1)            # rank 1 is the slow one
        nbytes = 1e9 * (rank + 1)
        out[rank] = (bench.reduce_max(ms, world), bench.reduce_sum(nbytes, world),
                     bench.job_throughput(nbytes, ms, world))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_job_throughput():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_rank, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
        got = dict(out)
    assert set(got) == {0, 1}
    for rank in (0, 1):
        mx, total, gbs = got[rank]
        assert mx == 20.0 and total == 3e9
        assert abs(gbs - 3e9 / 20e-3 / 1e9) < 1e-9  # 150 GB/s over the slowest rank's 20 ms


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.5, 1) == 3.5 and bench.reduce_sum(2.0, 1) == 2.0
    assert abs(bench.job_throughput(6e9, 2.0, 1) - 3000.0) < 1e-9
    bench.barrier(1)
