"""One rank of the context-parallel ring on its own GPU.

Page "序列与上下文并行", section "上下文并行：注意力本身切分": every rank keeps its
Q/K/V chunk, the K/V blocks travel around the ring one step at a time, and each
rank computes on the block it holds while the next one arrives; the per-step
partials are merged by online softmax. At step t rank r works on the block of
rank (r + t) mod N, so the block it needs next is the one the next rank,
r + 1, holds at the same step: each rank pulls it from there.

On B200 a rank's two receive slots (K and V of one block each) are device
buffers the neighbour's process maps through CUDA IPC. The pull is a copy-engine
transfer over NVLink (``cp_copy_async``) on a side stream, so it overlaps the
step's attention kernel without taking its SMs, and the kernel reads keys and
values from local HBM only. No kernel waits on another GPU: the order between
ranks is kept on the host, by events and a host barrier per step (``run_ring``).
"""
from __future__ import annotations

import ctypes
import threading
from typing import Callable, Optional, Sequence

import torch

from . import (DeviceBuffer, PeerBuffer, Plan, _check, attn_fwd_ring_step, copy_async, lib,
               merge_partials)


def run_ring(n: int, compute: Callable[[int], None], pull: Callable[[int], None],
             wait_pull: Callable[[int], None], wait_compute: Callable[[int], None],
             barrier: Callable[[], None], wait_fill: Callable[[], None]) -> None:
    """Drive one rank through the N steps of a ring forward.

    Slots: slot s of a rank holds one K/V block; at step t the rank's block
    (rank + t) mod N is in its slot t % 2 (its own block for t = 0, copied there
    by the caller before the call: the fill).

      compute(t)       enqueue step t's attention; t >= 1 reads slot t % 2 and must
                       be ordered after pull(t - 1) on the device
      pull(t)          enqueue the copy of the next rank's slot t % 2 into this
                       rank's slot (t + 1) % 2: block (rank + t + 1) mod N
      wait_pull(t), wait_compute(t), wait_fill()
                       block the host until that operation has finished
      barrier()        host barrier of all ranks of the ring

    pull(t + 1) overwrites this rank's slot t % 2 and reads the next rank's slot
    (t + 1) % 2. Before it is issued: this rank's compute(t) has finished (its
    last reader here); the previous rank's pull(t), which read it, has finished;
    and the next rank's pull(t), which filled the slot read, has finished. Each
    rank waits for its own pull(t) and compute(t) and then meets the others at a
    barrier, which gives all three. The final barrier leaves no rank reading
    another's slots when the call returns, so the next call may refill them.
    """
    compute(0)          # the rank's own block: no dependency on any peer
    wait_fill()         # slot 0 holds the own block for the previous rank to read
    barrier()
    if n > 1:
        pull(0)
    for t in range(n - 1):
        compute(t + 1)                 # ordered after pull(t)
        if t + 1 < n - 1:
            wait_pull(t)
            wait_compute(t)
            barrier()
            pull(t + 1)
    if n > 1:
        wait_pull(n - 2)
        barrier()


class RingRank:
    """Forward attention of one rank of the ring (contiguous or zigzag layout).

    ``plan`` describes the whole problem (B, H, S, D, N, causal, layout); this rank
    holds tokens of its chunk in the layout's local order (zigzag: chunks r and
    2N - 1 - r of 2N). ``barrier`` is the host barrier of all ranks. After
    ``connect`` with the next rank's slot buffer (``next_slots_ptr`` is its base
    pointer in this process), ``forward`` returns the rank's rows of full softmax
    attention.
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
        # slot s: K at s * 2 * block_bytes, V right after it
        self.slots = DeviceBuffer(4 * self.block_bytes)
        self.next_slots_ptr: Optional[int] = None
        self.o_parts = torch.empty(N, self.rows, D, dtype=torch.float32, device=self.device)
        self.lse_parts = torch.empty(N, self.rows, dtype=torch.float32, device=self.device)
        self.copy_stream = torch.cuda.Stream(device=self.device)
        self.fill_done = torch.cuda.Event()
        self.pull_done = [torch.cuda.Event() for _ in range(max(N - 1, 1))]
        self.compute_done = [torch.cuda.Event() for _ in range(N)]
        plan.ring_prepare(self.rank)

    def slot_ptrs(self, s: int):
        base = self.slots.ptr + s * 2 * self.block_bytes
        return base, base + self.block_bytes

    def slot_kv(self, s: int):
        """Views of slot s as (K, V) tensors [B, S/N, H, D] bf16."""
        kp, vp = self.slot_ptrs(s)
        return (self.slots.view(self.shape, torch.bfloat16, kp - self.slots.ptr, self.device),
                self.slots.view(self.shape, torch.bfloat16, vp - self.slots.ptr, self.device))

    def ipc_handle(self) -> bytes:
        return self.slots.ipc_handle()

    def connect(self, next_slots_ptr: int):
        self.next_slots_ptr = int(next_slots_ptr)

    def forward(self, q, k, v, stream=None):
        """Rank-local q, k, v [B, S/N, H, D] bf16 -> (o [B, S/N, H, D] bf16,
        lse [rows] fp32 with row = (b*(S/N) + tl)*H + h)."""
        if self.next_slots_ptr is None and self.plan.N > 1:
            raise RuntimeError("RingRank.connect() has not been called")
        for x in (q, k, v):
            if x.dtype != torch.bfloat16 or tuple(x.shape) != self.shape or not x.is_contiguous():
                raise ValueError(f"expected contiguous bf16 {self.shape}")
        N, st = self.plan.N, stream if stream is not None else torch.cuda.current_stream(self.device)
        cs = self.copy_stream
        k0, v0 = self.slot_ptrs(0)
        copy_async(k0, k.data_ptr(), self.block_bytes, st)
        copy_async(v0, v.data_ptr(), self.block_bytes, st)
        self.fill_done.record(st)

        def compute(t):
            if t == 0:
                kp, vp = k.data_ptr(), v.data_ptr()
            else:
                st.wait_event(self.pull_done[t - 1])
                kp, vp = self.slot_ptrs(t % 2)
            _check("cp_attn_fwd_ring_step",
                   lib().cp_attn_fwd_ring_step(self.plan.handle, self.rank, t, _vp(q.data_ptr()), _vp(kp), _vp(vp),
                                               _vp(self.o_parts[t].data_ptr()), _vp(self.lse_parts[t].data_ptr()),
                                               _vp(st.cuda_stream)))
            self.compute_done[t].record(st)

        def pull(t):
            cs.wait_event(self.fill_done)
            if t >= 1:
                cs.wait_event(self.compute_done[t - 1])
            src = self.next_slots_ptr + (t % 2) * 2 * self.block_bytes
            dst = self.slots.ptr + ((t + 1) % 2) * 2 * self.block_bytes
            copy_async(dst, src, 2 * self.block_bytes, cs)
            self.pull_done[t].record(cs)

        run_ring(N, compute, pull,
                 wait_pull=lambda t: self.pull_done[t].synchronize(),
                 wait_compute=lambda t: self.compute_done[t].synchronize(),
                 barrier=self.barrier, wait_fill=self.fill_done.synchronize)
        o, lse = merge_partials(self.o_parts, self.lse_parts, stream=st)
        return o.view(self.shape), lse

    def close(self):
        self.slots.close()


def _vp(x: int):
    return ctypes.c_void_p(int(x))


def thread_ring(plan: Plan, timeout: float = 60.0):
    """The ring of one process (the emulation on one GPU): N ranks sharing a host
    barrier, rank r pulling from rank r + 1's slots directly."""
    b = threading.Barrier(plan.N, timeout=timeout)
    ranks = [RingRank(plan, r, barrier=b.wait) for r in range(plan.N)]
    for r, rr in enumerate(ranks):
        rr._thread_barrier = b
        rr.connect(ranks[(r + 1) % plan.N].slots.ptr)
    return ranks


class IpcRing:
    """The multi-process ring: one process per GPU, ``torch.distributed`` for the
    handle exchange and the host barrier (a gloo group, so that the barrier never
    waits on a GPU). Each rank maps the next rank's slots through CUDA IPC."""

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
        self.peer = None
        if world > 1:
            self.peer = PeerBuffer(handles[(rank + 1) % world], 4 * self.rank_state.block_bytes)
            self.rank_state.connect(self.peer.ptr)
        dist.barrier(group=self.group)

    def forward(self, q, k, v, stream=None):
        return self.rank_state.forward(q, k, v, stream)

    def close(self):
        # every rank unmaps its peer before any rank frees the memory mapped
        if self.peer is not None:
            self.peer.close()
        self.dist.barrier(group=self.group)
        self.rank_state.close()


def run_threads(ranks: Sequence[RingRank], inputs: Sequence[tuple], timeout: float = 120.0):
    """Runs ``forward`` of every rank of ``thread_ring`` in its own host thread and
    compute stream; returns the per-rank (o, lse), ordered before the caller's
    current stream's later work."""
    out: list = [None] * len(ranks)
    errors: list = []
    caller = torch.cuda.current_stream()
    streams = [torch.cuda.Stream(device=rr.device) for rr in ranks]
    for s_ in streams:
        s_.wait_stream(caller)

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
    for s_ in streams:
        caller.wait_stream(s_)
    return out
