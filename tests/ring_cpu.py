"""A CPU model of one ring rank, for testing the ring protocol (``run_ring``)
without a GPU.

Each rank has two single-thread executors standing in for its compute and copy
streams (work runs in submission order on each; a task may wait on another
stream's future, like a stream waiting on an event), two receive slots holding a
K/V block each, and a tag per slot naming the block it holds. Compute checks the
tag of the slot it reads and computes the oracle partial; a pull checks the tag
of the peer slot it copies before and after the copy (so a peer overwriting it
mid-copy is caught) and sets its own slot's tag. Random sleeps in every task
shake the interleavings.
"""
from __future__ import annotations

import random
import time
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from context_long_sequence_cp_b200.ring import run_ring
from oracle.attention import merge, partial


class CpuRank:
    def __init__(self, rank, N, q, k, v, qpos, pos_of, causal, scale, slots, tags, barrier, seed=0,
                 jitter=0.002):
        """q, k, v: the rank's local [T, H, D] fp64 arrays; qpos [T] their global
        positions; pos_of(block) the positions of block ``block``'s tokens; slots
        [2, 2, T, H, D] and tags [2] arrays of this rank (shared with the previous
        rank); barrier() the host barrier."""
        self.rank, self.N = rank, N
        self.q, self.k, self.v, self.qpos, self.pos_of = q, k, v, qpos, pos_of
        self.causal, self.scale = causal, scale
        self.slots, self.tags, self.barrier = slots, tags, barrier
        self.rng = random.Random(seed * 1000 + rank)
        self.jitter = jitter
        self.errors = []

    def _sleep(self):
        time.sleep(self.rng.random() * self.jitter)

    def forward(self, next_slots, next_tags):
        N, r = self.N, self.rank
        comp, copy = ThreadPoolExecutor(1), ThreadPoolExecutor(1)
        parts = [None] * N
        pull_done = [None] * max(N - 1, 1)
        compute_done = [None] * N

        def fill_task():
            self._sleep()
            self.slots[0, 0] = self.k
            self.slots[0, 1] = self.v
            self.tags[0] = r

        fill_done = comp.submit(fill_task)

        def compute(t):
            def task():
                if t > 0:
                    pull_done[t - 1].result()
                self._sleep()
                blk = (r + t) % N
                if t == 0:
                    kk, vv = self.k, self.v
                else:
                    if int(self.tags[t % 2]) != blk:
                        self.errors.append(f"rank {r} step {t}: slot holds {int(self.tags[t % 2])}, wants {blk}")
                    kk, vv = self.slots[t % 2, 0].copy(), self.slots[t % 2, 1].copy()
                T, H, D = self.q.shape
                o = np.zeros((T, H, D))
                lse = np.zeros((T, H))
                for h in range(H):
                    o[:, h], lse[:, h] = partial(self.q[:, h], self.qpos, kk[:, h], vv[:, h], self.pos_of(blk),
                                                 causal=self.causal, scale=self.scale)
                parts[t] = (o.reshape(T * H, D), lse.reshape(T * H))
            compute_done[t] = comp.submit(task)

        def pull(t):
            def task():
                fill_done.result()
                if t >= 1:
                    compute_done[t - 1].result()
                want = (r + t + 1) % N
                if int(next_tags[t % 2]) != want:
                    self.errors.append(f"rank {r} pull {t}: peer slot holds {int(next_tags[t % 2])}, wants {want}")
                buf = next_slots[t % 2].copy()
                self._sleep()
                if int(next_tags[t % 2]) != want:
                    self.errors.append(f"rank {r} pull {t}: peer slot overwritten during the copy")
                self.slots[(t + 1) % 2] = buf
                self.tags[(t + 1) % 2] = want
            pull_done[t] = copy.submit(task)

        try:
            run_ring(N, compute, pull, wait_pull=lambda t: pull_done[t].result(),
                     wait_compute=lambda t: compute_done[t].result(), barrier=self.barrier,
                     wait_fill=fill_done.result)
            for f in compute_done:
                f.result()
        finally:
            comp.shutdown(wait=True)
            copy.shutdown(wait=True)
        return merge(parts)
