"""A CPU model of one ring rank, for testing the ring protocol (``run_ring``)
without a GPU.

Each rank has a single-thread executor standing in for its stream and another
for its copy stream, slot sets (set s, slot j: rank j's K/V block as fetched in a
call that used set s; slot ``rank`` is filled with the rank's own block), and a
tag per slot naming the (call, block) it holds. The forward runs as one task on
the rank's stream, like the persistent kernel: a copier thread (the copy warps)
fetches the other ranks' own blocks in ring order, checking each owner's slot tag
before and after the copy (so a refill during the copy is caught), and raises a
per-block arrival count; the units, step-major, wait (bounded) for their block's
arrival, check the slot's tag and compute the oracle partial. The fill runs on
the copy stream after everything on the rank's stream. Random sleeps shake the
interleavings, and a rank can be given a slow copier, so that the others run
ahead.
"""
from __future__ import annotations

import random
import threading
import time
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from context_long_sequence_cp_b200.ring import SLOT_SETS, run_ring
from oracle.attention import merge, partial


class CpuRank:
    def __init__(self, rank, N, q, k, v, qpos, pos_of, causal, scale, slots, tags, barrier, seed=0,
                 jitter=0.002, pull_delay=0.0, sets=SLOT_SETS, fill_after_forward=True):
        """q, k, v: the rank's local [T, H, D] fp64 arrays; qpos [T] their global
        positions; pos_of(block) the positions of block ``block``'s tokens; slots
        [sets, N, 2, T, H, D] and tags [sets, N] (int64) arrays of this rank,
        readable by the other ranks; barrier() the host barrier."""
        self.rank, self.N = rank, N
        self.q, self.k, self.v, self.qpos, self.pos_of = q, k, v, qpos, pos_of
        self.causal, self.scale = causal, scale
        self.slots, self.tags, self.barrier = slots, tags, barrier
        self.sets, self.fill_after_forward = sets, fill_after_forward
        self.calls = 0
        self.rng = random.Random(seed * 1000 + rank)
        self.jitter = jitter
        self.pull_delay = pull_delay      # extra time each fetched block takes (a slow link)
        self.errors = []
        self.stream = ThreadPoolExecutor(1)
        self.copy_stream = ThreadPoolExecutor(1)
        self.last = None

    def _sleep(self):
        time.sleep(self.rng.random() * self.jitter)

    def close(self):
        self.stream.shutdown(wait=True)
        self.copy_stream.shutdown(wait=True)

    def forward(self, peer_slots, peer_tags):
        """peer_slots[j], peer_tags[j]: rank j's slot and tag arrays (own included).
        Returns a future of (O, lse)."""
        N, r = self.N, self.rank
        c = self.calls
        self.calls += 1
        sset = c % self.sets
        tag = lambda j: c * N + j
        prev = self.last

        def fill_task():
            if prev is not None and self.fill_after_forward:
                prev.result()                     # stream order: after the previous forward
            self._sleep()
            self.slots[sset, r, 0] = self.k
            self.slots[sset, r, 1] = self.v
            self.tags[sset, r] = tag(r)

        fill_done = []

        def forward_task():
            arrived = np.zeros(N, dtype=np.int64)

            def copier():
                for t in range(1, N):
                    j = (r + t) % N
                    if int(peer_tags[j][sset, j]) != tag(j):
                        self.errors.append(f"rank {r} call {c}: owner {j}'s slot holds {int(peer_tags[j][sset, j])}")
                    buf = peer_slots[j][sset, j].copy()
                    self._sleep()
                    time.sleep(self.pull_delay)
                    if int(peer_tags[j][sset, j]) != tag(j):
                        self.errors.append(f"rank {r} call {c}: owner {j}'s slot refilled during the copy")
                    self.slots[sset, j] = buf
                    self.tags[sset, j] = tag(j)
                    arrived[j] = 1

            th = threading.Thread(target=copier)
            th.start()
            parts = []
            T, H, D = self.q.shape
            for t in range(N):
                j = (r + t) % N
                if t > 0:
                    t0 = time.monotonic()
                    while not arrived[j]:
                        if time.monotonic() - t0 > 30:
                            raise TimeoutError(f"rank {r}: block {j} never arrived")
                        time.sleep(1e-4)
                if int(self.tags[sset, j]) != tag(j):
                    self.errors.append(f"rank {r} call {c} step {t}: slot {j} holds {int(self.tags[sset, j])}")
                kk, vv = self.slots[sset, j, 0].copy(), self.slots[sset, j, 1].copy()
                o = np.zeros((T, H, D))
                lse = np.zeros((T, H))
                for h in range(H):
                    o[:, h], lse[:, h] = partial(self.q[:, h], self.qpos, kk[:, h], vv[:, h], self.pos_of(j),
                                                 causal=self.causal, scale=self.scale)
                parts.append((o.reshape(T * H, D), lse.reshape(T * H)))
            th.join()
            return merge(parts)

        def fill():
            fill_done.append(self.copy_stream.submit(fill_task))

        def launch():
            f = fill_done[0]
            self.last = self.stream.submit(lambda: (f.result(), forward_task())[1])

        run_ring(fill, lambda: fill_done[0].result(), self.barrier, launch)
        return self.last
