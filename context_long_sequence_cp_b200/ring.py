"""One rank of the context-parallel ring on its own GPU.

Page "序列与上下文并行", section "上下文并行：注意力本身切分": every rank keeps its
Q/K/V chunk, the K/V blocks of the other ranks reach it one ring step at a time,
and it computes on the blocks it holds while the next ones arrive; the per-step
partials are merged by online softmax. At step t rank r works on the block of
rank (r + t) mod N.

B200 design. Behind NVSwitch every GPU reaches every other at full NVLink
bandwidth, so rank r fetches block (r + t) mod N straight from its owner rather
than having it relayed hop by hop: the same bytes per rank (N - 1 blocks), no
chain of per-step hand-offs. Each rank exposes its own block in a slot buffer
the others map through CUDA IPC. The whole forward is ONE persistent,
cooperative kernel launch (``cp_attn_fwd_ring``): the first half of the ring
steps runs step-major, one unit per (step, query-tile pair), starting on the
rank's own block; then each pair walks the remaining steps in one unit. Two
copy warps of every CTA meanwhile load the other blocks over NVLink, in ring
order, into local slots, publishing per-block arrival counts that the units
wait on. The transfer overlaps the math inside one
kernel and needs no copy engine, stream or event between them (a device-to-device
copy issued on another stream does not progress while the persistent kernel
holds every SM). The ranks meet at ONE host barrier per call, after every rank's
own block is in place. Slot buffers alternate between calls, so that a rank may
refill its own block while the others still read the previous call's.
"""
from __future__ import annotations

import ctypes
import threading
from typing import Callable, Optional, Sequence

import torch

from . import DeviceBuffer, PeerBuffer, Plan, _check, copy_async, lib, merge_partials

SLOT_SETS = 2   # call c uses slot set c mod 2


def run_ring(fill: Callable[[], None], wait_fill: Callable[[], None], barrier: Callable[[], None],
             launch: Callable[[], None]) -> None:
    """Drive one rank through a ring forward (call c, slot set c mod 2).

    ``fill()`` enqueues the copy of the rank's own block into its slot of this
    call's set, ordered on the device after everything before it on the rank's
    stream, the rank's forward of call c - 1 included; ``wait_fill()`` blocks the
    host until the fill has finished; ``barrier()`` is the host barrier of all
    ranks; ``launch()`` enqueues the forward, which fetches the other ranks' own
    blocks of this call's set.

    After the barrier every rank's own block of set c mod 2 is in place, and every
    rank's fill of call c has finished, hence (device order) its forward of call
    c - 1: no forward still reads set (c + 1) mod 2, which call c + 1 refills
    (after this barrier, in host order). One barrier per call.
    """
    fill()
    wait_fill()
    barrier()
    launch()


class RingRank:
    """Forward attention of one rank of the ring (contiguous or zigzag layout).

    ``plan`` describes the whole problem (B, H, S, D, N, causal, layout); this rank
    holds the tokens of its chunk in the layout's local order (zigzag: chunks r
    and 2N - 1 - r of 2N). ``barrier`` is the host barrier of all ranks. After
    ``connect`` with every rank's slot buffer as mapped in this process,
    ``forward`` returns the rank's rows of full softmax attention. Successive
    calls of one rank go on one stream.
    """

    def __init__(self, plan: Plan, rank: int, barrier: Callable[[], None], device=None):
        if plan.layout == "ulysses":
            raise ValueError("the ring runs the contiguous and zigzag layouts")
        self.plan, self.rank, self.barrier = plan, int(rank), barrier
        self.device = torch.device(device) if device is not None else torch.device("cuda",
                                                                                     torch.cuda.current_device())
        B, H, S, D, N = plan.B, plan.H, plan.S, plan.D, plan.N
        self.T = S // N
        self.shape = (B, self.T, H, D)
        self.rows = B * self.T * H
        self.block_bytes = B * self.T * H * D * 2
        self.set_bytes = 2 * N * self.block_bytes
        # SLOT_SETS sets of [K of every rank's block [N][B][S/N][H][D], then V]
        self.slots = DeviceBuffer(SLOT_SETS * self.set_bytes)
        self.peer_bases: Optional[list] = None
        self.arrived = torch.zeros(N, dtype=torch.int32, device=self.device)
        P = plan.ring_parts()
        self.o_parts = torch.empty(P, self.rows, D, dtype=torch.float32, device=self.device)
        self.lse_parts = torch.empty(P, self.rows, dtype=torch.float32, device=self.device)
        self.calls = 0
        self.copy_stream = torch.cuda.Stream(device=self.device)
        self.fill_done = torch.cuda.Event()
        plan.ring_prepare(self.rank)

    def set_ptrs(self, base: int, c: int):
        """(K, V) slot-array addresses of call c's set in a slot buffer at base."""
        k = base + (c % SLOT_SETS) * self.set_bytes
        return k, k + self.plan.N * self.block_bytes

    def ipc_handle(self) -> bytes:
        return self.slots.ipc_handle()

    def connect(self, peer_bases: Sequence[int]):
        """peer_bases[j]: rank j's slot buffer as mapped in this process."""
        if len(peer_bases) != self.plan.N:
            raise ValueError("one slot buffer per rank")
        self.peer_bases = [int(b) for b in peer_bases]

    def pull_sources(self, c: int):
        """Device addresses of every rank's own K and V block of call c's set."""
        ks, vs = [], []
        for j, base in enumerate(self.peer_bases):
            k, v = self.set_ptrs(base, c)
            ks.append(k + j * self.block_bytes)
            vs.append(v + j * self.block_bytes)
        return ks, vs

    def forward(self, q, k, v, stream=None):
        """Rank-local q, k, v [B, S/N, H, D] bf16 -> (o [B, S/N, H, D] bf16,
        lse [rows] fp32 with row = (b*(S/N) + tl)*H + h)."""
        N, r = self.plan.N, self.rank
        if self.peer_bases is None:
            raise RuntimeError("RingRank.connect() has not been called")
        for x in (q, k, v):
            if x.dtype != torch.bfloat16 or tuple(x.shape) != self.shape or not x.is_contiguous():
                raise ValueError(f"expected contiguous bf16 {self.shape}")
        st = stream if stream is not None else torch.cuda.current_stream(self.device)
        cs = self.copy_stream
        c = self.calls
        self.calls += 1
        k_all, v_all = self.set_ptrs(self.slots.ptr, c)

        def fill():
            cs.wait_stream(st)          # k and v are ready; the forward of call c - 1 is done
            copy_async(k_all + r * self.block_bytes, k.data_ptr(), self.block_bytes, cs)
            copy_async(v_all + r * self.block_bytes, v.data_ptr(), self.block_bytes, cs)
            self.fill_done.record(cs)

        def launch():
            st.wait_event(self.fill_done)
            pk, pv = self.pull_sources(c) if N > 1 else (None, None)
            _launch_ring(self.plan, r, q, k_all, v_all, pk, pv, self.arrived if N > 1 else None, self.o_parts,
                         self.lse_parts, st)

        run_ring(fill, self.fill_done.synchronize, self.barrier, launch)
        o, lse = merge_partials(self.o_parts, self.lse_parts, stream=st)
        return o.view(self.shape), lse

    def close(self):
        self.slots.close()


def _launch_ring(plan, rank, q, k_all, v_all, pk, pv, arrived, o_parts, lse_parts, st):
    if pk is None:
        pka = pva = None
    else:
        pka = ctypes.cast((ctypes.c_void_p * len(pk))(*pk), ctypes.c_void_p)
        pva = ctypes.cast((ctypes.c_void_p * len(pv))(*pv), ctypes.c_void_p)
    _check("cp_attn_fwd_ring",
           lib().cp_attn_fwd_ring(plan.handle, rank, _vp(q.data_ptr()), _vp(k_all), _vp(v_all), pka, pva,
                                  None if arrived is None else _vp(arrived.data_ptr()), _vp(o_parts.data_ptr()),
                                  _vp(lse_parts.data_ptr()),
                                  _vp(st.cuda_stream)))


def _vp(x: int):
    return ctypes.c_void_p(int(x))


def thread_ring(plan: Plan, timeout: float = 60.0):
    """The ring of one process (the emulation on one GPU): N ranks sharing a host
    barrier, each pulling from the others' slot buffers directly."""
    b = threading.Barrier(plan.N, timeout=timeout)
    ranks = [RingRank(plan, r, barrier=b.wait) for r in range(plan.N)]
    for rr in ranks:
        rr._thread_barrier = b
        rr.connect([x.slots.ptr for x in ranks])
    return ranks


class IpcRing:
    """The multi-process ring: one process per GPU, ``torch.distributed`` for the
    handle exchange and the host barrier (a gloo group, so that the barrier never
    waits on a GPU). Each rank maps every other rank's slot buffer through CUDA
    IPC (NVSwitch: all pairs at full bandwidth)."""

    def __init__(self, plan: Plan, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group if group is not None else dist.new_group(backend="gloo")
        rank, world = dist.get_rank(self.group), dist.get_world_size(self.group)
        if world != plan.N:
            raise ValueError(f"the ring has {world} ranks, the plan {plan.N}")
        self.rank_state = RingRank(plan, rank, barrier=lambda: dist.barrier(group=self.group))
        handles: list = [None] * world
        dist.all_gather_object(handles, self.rank_state.ipc_handle(), group=self.group)
        nbytes = SLOT_SETS * self.rank_state.set_bytes
        self.peers = {j: PeerBuffer(handles[j], nbytes) for j in range(world) if j != rank}
        self.rank_state.connect([self.rank_state.slots.ptr if j == rank else self.peers[j].ptr
                                 for j in range(world)])
        dist.barrier(group=self.group)

    def forward(self, q, k, v, stream=None):
        return self.rank_state.forward(q, k, v, stream)

    def close(self):
        # every rank unmaps its peers before any rank frees the memory they map
        for pb in self.peers.values():
            pb.close()
        self.dist.barrier(group=self.group)
        self.rank_state.close()


def run_threads(ranks: Sequence[RingRank], inputs: Sequence[tuple], timeout: float = 120.0):
    """Runs ``forward`` of every rank of ``thread_ring`` in its own host thread;
    returns the per-rank (o, lse), ordered before the caller's current stream's
    later work. The ranks' launches share one stream: on one GPU the cooperative
    launches of different ranks must not be resident at the same time."""
    out: list = [None] * len(ranks)
    errors: list = []
    caller = torch.cuda.current_stream()
    shared = torch.cuda.Stream(device=ranks[0].device)
    shared.wait_stream(caller)
    streams = [shared] * len(ranks)

    def body(r):
        try:
            with torch.cuda.device(ranks[r].device):
                out[r] = ranks[r].forward(*inputs[r], stream=streams[r])
        except BaseException as e:  # noqa: BLE001 - re-raised in the caller
            errors.append(e)
            b = getattr(ranks[r], "_thread_barrier", None)
            if b is not None:
                b.abort()

    threads = [threading.Thread(target=body, args=(r,)) for r in range(len(ranks))]
    for th in threads:
        th.start()
    for th in threads:
        th.join(timeout)
    if any(th.is_alive() for th in threads):
        raise TimeoutError("ring threads did not finish")
    if errors:
        raise errors[0]
    caller.wait_stream(shared)
    return out
