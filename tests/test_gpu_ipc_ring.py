"""The multi-process ring on one GPU: one process per rank, CUDA IPC, gloo.

Every rank is its own process (spawned), as on N GPUs: it allocates its slot
buffer, exchanges IPC handles with the others (``IpcRing``), maps every peer's
buffer with ``cp_ipc_open_handle``, fills its own block, meets the others at the
host barrier, and runs its one-launch ring forward, whose copy warps read the
peers' own blocks through the mapped pointers. Only one GPU is available here,
so the ranks take turns to launch (extra gloo barriers after the protocol's
own), and no two cooperative grids are ever resident together; no kernel waits
on another process's kernel (a rank's units wait only for its own copy warps,
and the peers' blocks are in place before the barrier). Three calls in a row
exercise both slot sets and their reuse. Each rank's outputs must be
bit-identical to the same rank of the one-process ring (``thread_ring``) on the
same inputs, its pulled slots bit-identical to the peers' blocks; the handles
are then closed in ``IpcRing.close``'s order (every rank unmaps its peers before
any rank frees its buffer).
"""
import datetime
import os
import socket

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CALLS = 3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_inputs(shape, seed, rank):
    from tests import gpu_util as G
    from workloads import make_small
    B, H, S, D, N, layout, causal = shape
    q, k, v = make_small(B, H, S, D, seed)
    return [G.to_layout(x, N, layout)[rank].contiguous() for x in (q, k, v)], (q, k, v)


def _child(rank, world, port, shape, seed, out_q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=90))
    try:
        torch.cuda.set_device(0)
        import context_long_sequence_cp_b200 as cp
        from context_long_sequence_cp_b200 import ring as R
        B, H, S, D, N, layout, causal = shape
        plan = cp.Plan(B, H, S, D, N, causal, layout)
        (q, k, v), _ = _rank_inputs(shape, seed, rank)
        q, k, v = q.cuda(), k.cuda(), v.cuda()
        ring = R.IpcRing(plan)
        rs = ring.rank_state
        base = rs.barrier

        def after_fill_wait_turn():
            base()                        # every rank's own block is in place
            for _ in range(rank):         # the ranks before this one launch first
                base()

        outs = []
        for _ in range(CALLS):
            rs.barrier = after_fill_wait_turn
            o, lse = rs.forward(q, k, v)
            torch.cuda.synchronize()
            rs.barrier = base
            for _ in range(rank, N - 1):  # let the later ranks launch
                base()
            status = cp.check(plan)
            # the pulled slots of this call's set against the peers' own blocks
            c = rs.calls - 1
            k_all, v_all = rs.set_ptrs(rs.slots.ptr, c)
            blk = (B, S // N, H, D)
            pulled = []
            for j in range(N):
                if j == rank:
                    continue
                (_, kj, vj), _ = _rank_inputs(shape, seed, j)
                ks = cp._device_view(k_all + j * rs.block_bytes, blk, torch.bfloat16).cpu()
                vs = cp._device_view(v_all + j * rs.block_bytes, blk, torch.bfloat16).cpu()
                pulled.append(torch.equal(ks.view(torch.int16), kj.view(torch.int16)) and
                              torch.equal(vs.view(torch.int16), vj.view(torch.int16)))
            outs.append((o.cpu(), lse.cpu(), status, all(pulled)))
        ring.close()
        out_q.put((rank, outs, None))
    except BaseException as e:  # noqa: BLE001 - reported to the parent
        out_q.put((rank, None, repr(e)))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("shape,seed", [
    ((1, 2, 1024, 128, 2, "zigzag", True), 301),
    ((1, 2, 1536, 64, 3, "contiguous", True), 302),
])
def test_ipc_ring_processes_match_thread_ring(shape, seed):
    import torch.multiprocessing as mp
    import context_long_sequence_cp_b200 as cp
    from context_long_sequence_cp_b200 import ring as R
    B, H, S, D, N, layout, causal = shape
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_child, args=(r, N, port, shape, seed, q_out)) for r in range(N)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(N):
        rank, outs, err = q_out.get(timeout=240)
        assert err is None, f"rank {rank}: {err}"
        results[rank] = outs
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    # the same ring in one process: N ranks as host threads, launches on one stream
    plan = cp.Plan(B, H, S, D, N, causal, layout)
    ranks = R.thread_ring(plan)
    inputs = [tuple(x.cuda() for x in _rank_inputs(shape, seed, r)[0]) for r in range(N)]
    ref = R.run_threads(ranks, inputs)
    torch.cuda.synchronize()
    assert cp.check(plan) == 0
    for r in range(N):
        o_ref, l_ref = (x.cpu() for x in ref[r])
        for call, (o, lse, status, pulled_ok) in enumerate(results[r]):
            assert status == 0, (r, call)
            assert pulled_ok, (r, call)
            assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16)), (r, call)
            assert torch.equal(lse.view(torch.int32), l_ref.view(torch.int32)), (r, call)
    for rr in ranks:
        rr.close()
