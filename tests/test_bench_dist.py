"""The multi-process (N > 1) host path of bench.py on CPU: gloo, world size 2.

Each rank runs an independent replica (weak scaling); the job time is the
maximum of the ranks' times and the value sums the ranks' work.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [10.0, 12.5][rank]                 # rank 1 is the slowest
        job_ms, tflops = bench.job_throughput(local_ms, 1e12, world)
        q.put((rank, job_ms, tflops, bench.dist_env()))
    finally:
        dist.destroy_process_group()


def test_job_throughput_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, job_ms, tflops, env in res:
        assert job_ms == 12.5                          # max over ranks
        assert abs(tflops - 2 * 1e12 / 12.5e-3 / 1e12) < 1e-9   # both ranks' work / job time
        assert env == (2, rank, rank)


def test_job_throughput_single_rank():
    import bench
    job_ms, tflops = bench.job_throughput(8.0, 8.796e12, 1)
    assert job_ms == 8.0 and abs(tflops - 8.796e12 / 8e-3 / 1e12) < 1e-9
