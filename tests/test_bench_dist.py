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


class _FakeEvent:
    """Host-clock stand-in for a CUDA event (record / elapsed_time in ms)."""

    def __init__(self):
        self.t = None

    def record(self):
        import time
        self.t = time.perf_counter()

    def elapsed_time(self, other):
        return (other.t - self.t) * 1e3


def _ring_worker(rank, world, port, q):
    import sys
    import time
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from workloads import WORKLOADS
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        calls = []
        barriers = []

        def step():                                   # the stubbed ring forward: rank 1 is slower
            calls.append(1)
            time.sleep(0.002 * (rank + 1))

        def barrier():
            barriers.append(len(calls))
            dist.barrier()

        local_ms = bench.timed_ring_steps(step, barrier, lambda: (_FakeEvent(), _FakeEvent()), steps=5, warmup=3)
        w = WORKLOADS["zigzag_32k"]
        job_ms, _ = bench.job_throughput(local_ms, w.flops / world, world)
        line = bench.ring_line(w, world, 5, 3, job_ms, local_ms, 7.0, job_ms * 2, 10, 20, {"sm_mhz": None}, 1700.0,
                               "measured")
        q.put((rank, len(calls), barriers, local_ms, job_ms, line))
    finally:
        dist.destroy_process_group()


def test_ring_mode_timing_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ring_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    ms = [r[3] for r in res]
    for rank, ncalls, barriers, local_ms, job_ms, line in res:
        assert ncalls == 3 + 5                        # warm-up + timed steps
        assert barriers == [3, 8]                     # one barrier before and one after the timed steps
        assert job_ms == max(ms)                      # the slowest rank's time
        assert local_ms >= 2.0 * (rank + 1) * 0.9
        assert line["scaling"] == "strong" and line["n_gpus"] == 2
        from workloads import WORKLOADS
        w = WORKLOADS["zigzag_32k"]
        assert abs(line["value"] - w.flops / (job_ms * 1e-3) / 1e12) < 1e-9   # the whole problem / job time
        assert line["config"]["N"] == 2 and line["config"]["workload"] == "zigzag_32k"
        assert abs(line["components"]["ring_overhead_vs_fused_share"] - (job_ms / 3.5 - 1)) < 1e-9
