"""Host-side checks of the multi-GPU ring (no GPU): the per-rank step schedules
of the C library, and the ring protocol (``run_ring``) on a CPU model of the
ranks' streams, as threads of one process and as gloo processes.

The protocol runs each rank on its own block first, pulls block (r + t + 1) mod N
from rank r + 1 while step t computes, and orders the ranks by host barriers
(page "序列与上下文并行", section "上下文并行：注意力本身切分": the K/V blocks
travel around the ring while each rank computes on the one it holds). The
result must equal full attention for every rank's rows (oracle).
"""
import ctypes
import os
import socket
import threading

import numpy as np
import pytest

import context_long_sequence_cp_b200 as cp
from context_long_sequence_cp_b200 import build as cpbuild
from oracle.attention import attention, default_scale
from oracle.layouts import chunk_positions


@pytest.fixture(scope="module", autouse=True)
def built():
    cpbuild.build()


# ------------------------------------------------------------------ schedules

def _step_walk_lengths(S, N, layout, causal, r, t, tile=128):
    """Key tiles walked by each query-tile pair of rank r at ring step t: a key
    tile of block (r + t) mod N counts when either query tile has an allowed key
    in it (brute force over the positions)."""
    pos = chunk_positions(S, N, layout)
    T = S // N
    nt = -(-T // tile)
    rk = (r + t) % N
    tiles = lambda rr: [pos[rr, i * tile:(i + 1) * tile] for i in range(nt)]
    qt, kt = tiles(r), tiles(rk)
    out = []
    for qp in range(-(-nt // 2)):
        n = 0
        for kk in kt:
            ok = False
            for qq in qt[2 * qp:2 * qp + 2]:
                ok |= (not causal) or bool(kk.min() <= qq.max())
            n += ok
        out.append(n)
    return out


@pytest.mark.parametrize("S,N,layout,causal,B,H", [
    (4096, 4, "zigzag", True, 1, 4),
    (2048, 4, "contiguous", True, 2, 2),
    (1024, 2, "contiguous", False, 1, 3),
    (3840, 5, "zigzag", True, 1, 2),      # ragged: 768 local tokens, pairs of 256
])
def test_ring_schedule_covers_every_item_once_with_its_step_walk(S, N, layout, causal, B, H):
    p = cp.Plan(B, H, S, 128, N, causal, layout)
    T = S // N
    npairs = -(-T // 256)
    for r in range(N):
        for t in range(N):
            items, loads = p.ring_schedule(r, t)
            assert len(items) == B * H * npairs
            keys = {(rb, h, qp) for rb, h, qp, _, _ in items}
            assert keys == {(r * B + b, h, qp) for b in range(B) for h in range(H) for qp in range(npairs)}
            walk = _step_walk_lengths(S, N, layout, causal, r, t)
            for rb, h, qp, cost, cta in items:
                assert cost == walk[qp]
            # CTAs run contiguous runs in order; loads are the model's 2 per key tile + 3 per item
            ctas = [it[4] for it in items]
            assert ctas == sorted(ctas)
            assert len(loads) == min(len(items), 148)
            assert sum(loads) == sum(2 * it[3] + 3 for it in items)


def test_ring_schedule_balance_zigzag_32k():
    p = cp.Plan(1, 32, 32768, 128, 8, True, "zigzag")
    for r in (0, 3, 7):
        for t in range(8):
            items, loads = p.ring_schedule(r, t)
            loads = np.array(loads)
            costs = np.array([2 * it[3] + 3 for it in items])
            # longest-first list scheduling: the tail is at most one item
            assert loads.max() <= loads.mean() + costs.max(), (r, t)
            if t > 0:
                # Off-diagonal steps carry the same work (zigzag balance) in one of two
                # shapes. Key rank above the query rank: the query pairs of the later
                # chunk see all 32 key tiles, those of the earlier chunk none (they
                # only write O = 0, lse = -inf), and 256 large items on 148 CTAs end
                # after two. Key rank below: every pair sees the block's earlier chunk,
                # 16 tiles, and 512 equal items take ceil(512 / 148) = 4 rounds.
                rk = (r + t) % 8
                if rk > r:
                    assert sorted(set(it[3] for it in items)) == [0, 32]
                    assert loads.max() == 2 * (2 * 32 + 3)
                else:
                    assert sorted(set(it[3] for it in items)) == [16]
                    assert loads.max() == 4 * (2 * 16 + 3)
                assert loads.sum() == 256 * (2 * 32 + 3) + 256 * 3 or loads.sum() == 512 * (2 * 16 + 3)


def test_ring_argument_validation():
    p = cp.Plan(1, 2, 1024, 64, 4, True, "zigzag")
    L = cp.lib()
    assert L.cp_attn_ring_prepare(None, 0) == -1
    assert L.cp_attn_ring_prepare(p.handle, -1) == -1
    assert L.cp_attn_ring_prepare(p.handle, 4) == -1
    assert L.cp_attn_ring_prepare(p.handle, 3) == 0           # host schedules only without a device
    assert L.cp_attn_ring_schedule(p.handle, 0, 4, None, None) == -1
    assert L.cp_attn_ring_schedule(p.handle, 4, 0, None, None) == -1
    assert L.cp_attn_ring_schedule(p.handle, 1, 2, None, None) == 2   # 2 heads x 1 query-tile pair (T = 256)
    buf = ctypes.c_void_p(16)
    assert L.cp_attn_fwd_ring_step(p.handle, 0, 0, None, buf, buf, buf, buf, None) == -1
    assert L.cp_attn_fwd_ring_step(p.handle, 4, 0, buf, buf, buf, buf, buf, None) == -1
    assert L.cp_attn_fwd_ring_step(p.handle, 0, -1, buf, buf, buf, buf, buf, None) == -1
    assert L.cp_attn_fwd_ring_step(p.handle, 0, 0, ctypes.c_void_p(18), buf, buf, buf, buf, None) == -3
    u = cp.Plan(1, 4, 1024, 64, 2, False, "ulysses")
    assert L.cp_attn_ring_prepare(u.handle, 0) == -2
    assert L.cp_attn_fwd_ring_step(u.handle, 0, 0, buf, buf, buf, buf, buf, None) == -2
    assert L.cp_ipc_handle_bytes() == 64
    assert L.cp_ipc_get_handle(None, ctypes.create_string_buffer(64)) == -1
    assert L.cp_copy_async(None, None, 0, None) == 0
    assert L.cp_copy_async(None, buf, 16, None) == -1
    out = ctypes.c_void_p()
    assert L.cp_ring_buffer_alloc(0, ctypes.byref(out)) == -1
    assert L.cp_ring_buffer_free(None) == 0


# ------------------------------------------------------------------ protocol

def _problem(N, layout, causal, seed, B=1, H=2, D=8, C=8):
    S = 2 * N * C
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((S, H, D)) for _ in range(3))
    pos = chunk_positions(S, N, layout)
    o_ref, lse_ref = attention(q[None], k[None], v[None], causal=causal)
    return S, q, k, v, pos, o_ref[0], lse_ref[0]


def _check_rank(r, o, lse, pos, o_ref, lse_ref, H, D):
    T = pos.shape[1]
    np.testing.assert_allclose(o.reshape(T, H, D), o_ref[pos[r]], atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse.reshape(T, H), lse_ref[:, pos[r]].T, atol=1e-12, rtol=0)


@pytest.mark.parametrize("N,layout,causal", [(1, "zigzag", True), (2, "zigzag", True), (3, "contiguous", True),
                                             (4, "zigzag", True), (5, "contiguous", False)])
def test_ring_protocol_threads(N, layout, causal):
    from tests.ring_cpu import CpuRank
    H, D = 2, 8
    S, q, k, v, pos, o_ref, lse_ref = _problem(N, layout, causal, seed=N)
    T = S // N
    bar = threading.Barrier(N, timeout=60)
    slots = [np.zeros((2, 2, T, H, D)) for _ in range(N)]
    tags = [np.full(2, -1, dtype=np.int64) for _ in range(N)]
    ranks = [CpuRank(r, N, q[pos[r]], k[pos[r]], v[pos[r]], pos[r], lambda b: pos[b], causal, default_scale(D),
                     slots[r], tags[r], bar.wait, seed=N) for r in range(N)]
    for rep in range(2):                       # a second call reuses the slots
        out = [None] * N
        errs = []

        def body(r):
            try:
                out[r] = ranks[r].forward(slots[(r + 1) % N], tags[(r + 1) % N])
            except BaseException as e:  # noqa: BLE001
                errs.append(e)
                bar.abort()

        th = [threading.Thread(target=body, args=(r,)) for r in range(N)]
        for t_ in th:
            t_.start()
        for t_ in th:
            t_.join(120)
        assert not errs, errs
        for r in range(N):
            assert not ranks[r].errors, ranks[r].errors
            _check_rank(r, *out[r], pos, o_ref, lse_ref, H, D)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_worker(rank, world, port, prefix, layout, causal, q_out):
    import datetime
    import sys
    from multiprocessing import shared_memory
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist
    from tests.ring_cpu import CpuRank
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    shms = []
    try:
        H, D = 2, 8
        S, q, k, v, pos, o_ref, lse_ref = _problem(world, layout, causal, seed=7)
        T = S // world
        shape = (2, 2, T, H, D)
        nbytes = int(np.prod(shape)) * 8 + 16
        own = shared_memory.SharedMemory(name=f"{prefix}_{rank}", create=True, size=nbytes)
        shms.append(own)
        dist.barrier()
        peer = shared_memory.SharedMemory(name=f"{prefix}_{(rank + 1) % world}")
        shms.append(peer)
        view = lambda m: (np.ndarray(shape, np.float64, m.buf, 16), np.ndarray(2, np.int64, m.buf, 0))
        slots, tags = view(own)
        tags[:] = -1
        nslots, ntags = view(peer)
        dist.barrier()
        rr = CpuRank(rank, world, q[pos[rank]], k[pos[rank]], v[pos[rank]], pos[rank], lambda b: pos[b], causal,
                     default_scale(D), slots, tags, dist.barrier, seed=11)
        ok = True
        for _ in range(2):
            o, lse = rr.forward(nslots, ntags)
            try:
                _check_rank(rank, o, lse, pos, o_ref, lse_ref, H, D)
            except AssertionError:
                ok = False
        dist.barrier()
        q_out.put((rank, ok, list(rr.errors)))
        del slots, tags, nslots, ntags
    finally:
        for m in shms:
            m.close()
        if shms:
            try:
                dist.barrier()
            except Exception:
                pass
            shms[0].unlink()
        dist.destroy_process_group()


@pytest.mark.parametrize("world,layout", [(2, "zigzag"), (3, "contiguous")])
def test_ring_protocol_gloo_processes(world, layout):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    prefix = f"cpring{os.getpid()}_{port}"
    procs = [ctx.Process(target=_gloo_worker, args=(r, world, port, prefix, layout, True, q_out))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    res = sorted(q_out.get(timeout=10) for _ in range(world))
    for rank, ok, errors in res:
        assert ok and not errors, (rank, errors)
