"""Host-side checks of the multi-GPU ring (no GPU): the per-rank schedules of
the C library (per ring step, and the one-launch forward's units), and the ring
protocol (``run_ring``) on a CPU model of the ranks' streams and copy warps, as
threads of one process and as gloo processes.

The protocol fills each rank's own slot, meets the other ranks at one barrier,
and runs the forward, which fetches the other ranks' own blocks in ring order
while it computes (page "序列与上下文并行", section "上下文并行：注意力本身切分":
each rank computes on the blocks it holds while the next ones arrive). Calls
run back to back, alternating between two slot sets. The result must equal full
attention for every rank's rows (oracle), and no fetch may read a slot before
its owner filled it or while its owner refills it.
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


@pytest.mark.parametrize("S,N,layout,causal,B,H", [(4096, 4, "zigzag", True, 1, 4), (2048, 4, "contiguous", True, 2, 2),
                                                     (3840, 5, "zigzag", True, 1, 2)])
def test_ring_launch_units_cover_every_step_once(S, N, layout, causal, B, H):
    p = cp.Plan(B, H, S, 128, N, causal, layout)
    npairs = -(-(S // N) // 256)
    split = N if N <= 2 else (N + 1) // 2
    assert p.ring_parts() == (split + 1 if split < N else N)
    for r in range(N):
        units, loads = p.ring_schedule(r, -1)
        ranges = {}
        for rb, h, qp, cost, cta in units:
            t0, t1 = (qp >> 16) & 0xff, (qp >> 24) & 0xff
            ranges.setdefault((rb, h, qp & 0xffff), []).append((t0, t1))
            walks = [_step_walk_lengths(S, N, layout, causal, r, t)[qp & 0xffff] for t in range(t0, t1)]
            assert cost == sum(walks)
            # the first phase is one step per unit, the tail the remaining steps
            assert (t1 == t0 + 1 and t0 < split) or (t0 == split and t1 == N)
        assert set(ranges) == {(r * B + b, h, qp) for b in range(B) for h in range(H) for qp in range(npairs)}
        for rs in ranges.values():          # every step of every pair exactly once
            assert sorted(t for a, b in rs for t in range(a, b)) == list(range(N))
        # each CTA's units run phase by phase; CTAs are contiguous runs
        assert [u[4] for u in units] == sorted(u[4] for u in units)
        for c in set(u[4] for u in units):
            phases = [(u[2] >> 16) & 0xff for u in units if u[4] == c]
            assert phases == sorted(phases)
        assert sum(loads) == sum(2 * u[3] + 3 for u in units)
        assert max(loads) <= np.mean(loads) + max(2 * u[3] + 3 for u in units)


def test_ring_argument_validation():
    p = cp.Plan(1, 2, 1024, 64, 4, True, "zigzag")
    L = cp.lib()
    buf = ctypes.c_void_p(16)
    assert L.cp_attn_ring_prepare(None, 0) == -1
    assert L.cp_attn_ring_prepare(p.handle, -1) == -1
    assert L.cp_attn_ring_prepare(p.handle, 4) == -1
    assert L.cp_attn_ring_prepare(p.handle, 3) == 0           # host schedules only without a device
    assert L.cp_attn_ring_schedule(p.handle, 0, 4, None, None) == -1
    assert L.cp_attn_ring_schedule(p.handle, 0, -2, None, None) == -1
    assert L.cp_attn_ring_schedule(p.handle, 2, -1, None, None) == 3 * 2   # steps 0, 1 and the tail [2, 4)
    assert L.cp_attn_ring_num_parts(p.handle) == 3
    srcs = ctypes.cast((ctypes.c_void_p * 4)(16, 32, 48, 64), ctypes.c_void_p)
    bad_src = ctypes.cast((ctypes.c_void_p * 4)(16, 40, 48, 64), ctypes.c_void_p)
    null_src = ctypes.cast((ctypes.c_void_p * 4)(16, None, 48, 64), ctypes.c_void_p)
    ring = lambda *a: L.cp_attn_fwd_ring(p.handle, *a)
    assert ring(0, None, buf, buf, None, None, None, buf, buf, None) == -1
    assert ring(5, buf, buf, buf, None, None, None, buf, buf, None) == -1
    assert ring(0, buf, buf, buf, srcs, None, buf, buf, buf, None) == -1          # K sources without V
    assert ring(0, buf, buf, buf, srcs, srcs, None, buf, buf, None) == -1         # pulling needs arrived
    assert ring(0, buf, buf, buf, null_src, srcs, buf, buf, buf, None) == -1      # a missing source
    assert ring(0, buf, buf, buf, bad_src, srcs, buf, buf, buf, None) == -3       # a misaligned source
    # without pull sources an arrived buffer is refused (a stale one would stall
    # every unit until its wait runs out); the explicit external-arrival entry
    # takes it, and refuses a missing or misaligned one
    assert ring(0, buf, buf, buf, None, None, buf, buf, buf, None) == -1
    ext = lambda *a: L.cp_attn_fwd_ring_external(p.handle, *a)
    assert ext(0, buf, buf, buf, None, buf, buf, None) == -1
    assert ext(0, buf, buf, buf, ctypes.c_void_p(18), buf, buf, None) == -3
    assert ext(4, buf, buf, buf, buf, buf, buf, None) == -1
    big = cp.Plan(1, 2, 65 * 256, 64, 65, False, "contiguous")
    srcs65 = ctypes.cast((ctypes.c_void_p * 65)(*([16] * 65)), ctypes.c_void_p)
    assert L.cp_attn_fwd_ring(big.handle, 0, buf, buf, buf, srcs65, srcs65, buf, buf, buf, None) == -2
    assert L.cp_attn_ring_schedule(p.handle, 4, 0, None, None) == -1
    assert L.cp_attn_ring_schedule(p.handle, 1, 2, None, None) == 2   # 2 heads x 1 query-tile pair (T = 256)
    assert L.cp_attn_fwd_ring_step(p.handle, 0, 0, None, buf, buf, buf, buf, None) == -1
    assert L.cp_attn_fwd_ring_step(p.handle, 4, 0, buf, buf, buf, buf, buf, None) == -1
    assert L.cp_attn_fwd_ring_step(p.handle, 0, -1, buf, buf, buf, buf, buf, None) == -1
    assert L.cp_attn_fwd_ring_step(p.handle, 0, 0, ctypes.c_void_p(18), buf, buf, buf, buf, None) == -3
    u = cp.Plan(1, 4, 1024, 64, 2, False, "ulysses")
    assert L.cp_attn_ring_prepare(u.handle, 0) == -2
    assert L.cp_attn_fwd_ring_step(u.handle, 0, 0, buf, buf, buf, buf, buf, None) == -2
    assert L.cp_attn_fwd_ring(u.handle, 0, buf, buf, buf, None, None, None, buf, buf, None) == -2
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


def _thread_ring(N, layout, causal, sets=None, fill_after_forward=True, calls=3, slow_rank=0):
    from tests.ring_cpu import CpuRank
    from context_long_sequence_cp_b200.ring import SLOT_SETS
    sets = SLOT_SETS if sets is None else sets
    H, D = 2, 8
    S, q, k, v, pos, o_ref, lse_ref = _problem(N, layout, causal, seed=N)
    T = S // N
    bar = threading.Barrier(N, timeout=60)
    slots = [np.zeros((sets, N, 2, T, H, D)) for _ in range(N)]
    tags = [np.full((sets, N), -1, dtype=np.int64) for _ in range(N)]
    # one rank fetches slowly: the others run ahead into the next calls and would
    # refill their slots under its fetches if the protocol let them
    ranks = [CpuRank(r, N, q[pos[r]], k[pos[r]], v[pos[r]], pos[r], lambda b: pos[b], causal, default_scale(D),
                     slots[r], tags[r], bar.wait, seed=N, pull_delay=0.01 if r == slow_rank else 0.0, sets=sets,
                     fill_after_forward=fill_after_forward) for r in range(N)]
    outs = [[] for _ in range(N)]
    errs = []

    def body(r):
        try:
            futs = [ranks[r].forward(slots, tags) for _ in range(calls)]
            outs[r] = [f.result(timeout=60) for f in futs]
        except BaseException as e:  # noqa: BLE001
            errs.append(e)
            bar.abort()

    th = [threading.Thread(target=body, args=(r,)) for r in range(N)]
    for t_ in th:
        t_.start()
    for t_ in th:
        t_.join(120)
    for rr in ranks:
        rr.close()
    bad = []
    for r in range(N):
        bad += ranks[r].errors
        for o, lse in outs[r]:
            try:
                _check_rank(r, o, lse, pos, o_ref, lse_ref, H, D)
            except AssertionError:
                bad.append(f"rank {r}: wrong result")
    return errs, bad


@pytest.mark.parametrize("N,layout,causal", [(1, "zigzag", True), (2, "zigzag", True), (3, "contiguous", True),
                                             (4, "zigzag", True), (5, "contiguous", False)])
def test_ring_protocol_threads(N, layout, causal):
    errs, bad = _thread_ring(N, layout, causal)
    assert not errs, errs
    assert not bad, bad


def test_ring_protocol_checks_catch_a_reused_slot_set():
    # One slot set and a fill not ordered after the rank's previous forward: a
    # fast rank refills its block while the slow rank still fetches it. The
    # model must notice (this is what the two alternating sets prevent).
    errs, bad = _thread_ring(4, "zigzag", True, sets=1, fill_after_forward=False, calls=3, slow_rank=0)
    assert errs or bad


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
        from context_long_sequence_cp_b200.ring import SLOT_SETS
        shape = (SLOT_SETS, world, 2, T, H, D)
        nbytes = int(np.prod(shape)) * 8 + 8 * SLOT_SETS * world
        own = shared_memory.SharedMemory(name=f"{prefix}_{rank}", create=True, size=nbytes)
        shms.append(own)
        dist.barrier()
        view = lambda m: (np.ndarray(shape, np.float64, m.buf, 8 * SLOT_SETS * world),
                          np.ndarray((SLOT_SETS, world), np.int64, m.buf, 0))
        peers = {j: shared_memory.SharedMemory(name=f"{prefix}_{j}") for j in range(world) if j != rank}
        shms.extend(peers.values())
        slots, tags = view(own)
        tags[:] = -1
        all_slots, all_tags = [], []
        for j in range(world):
            sj, tj = (slots, tags) if j == rank else view(peers[j])
            all_slots.append(sj)
            all_tags.append(tj)
        dist.barrier()
        rr = CpuRank(rank, world, q[pos[rank]], k[pos[rank]], v[pos[rank]], pos[rank], lambda b: pos[b], causal,
                     default_scale(D), slots, tags, dist.barrier, seed=11, pull_delay=0.01 if rank == 0 else 0.0)
        ok = True
        futs = [rr.forward(all_slots, all_tags) for _ in range(3)]
        for f in futs:
            o, lse = f.result(timeout=60)
            try:
                _check_rank(rank, o, lse, pos, o_ref, lse_ref, H, D)
            except AssertionError:
                ok = False
        rr.close()
        dist.barrier()
        q_out.put((rank, ok, list(rr.errors)))
        del rr, slots, tags, all_slots, all_tags, sj, tj   # release the views before closing the segments
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
