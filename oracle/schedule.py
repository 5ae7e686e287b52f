"""Executed (query tile, key tile) pairs per virtual rank — test infrastructure only.

Source: "序列与上下文并行" (ai-infra-wiki), section "上下文并行：注意力本身切分":
at ring step t rank r computes its Q block against the K/V block of rank
(r + t) mod N; under causal masking segment i needs only segments <= i, and the
zigzag assignment balances the work (section "工程实践": without it half the
cards idle).

Brute force: a pair of 128-token tiles is executed iff at least one (query,
key) pair in it is allowed — any pair for non-causal attention, pos(key) <=
pos(query) for causal. The count per rank (summed over ring steps, per
(batch, head)) is the per-rank work of the method; max/mean over ranks is its
load imbalance.
"""
from __future__ import annotations

import numpy as np

from .layouts import chunk_positions

TILE = 128


def tile_pair_counts(S: int, N: int, layout: str, causal: bool, tile: int = TILE) -> np.ndarray:
    """int64 [N]: executed tile pairs of each rank (per batch and head).

    Every (query tile, ring step, key tile) triple is enumerated; a pair is
    executed iff min(key positions) <= max(query positions) (causal), always
    otherwise.
    """
    pos = chunk_positions(S, N, layout)            # [N, T]
    T = S // N
    nt = -(-T // tile)
    tmin = np.empty((N, nt), dtype=np.int64)
    tmax = np.empty((N, nt), dtype=np.int64)
    for r in range(N):
        for i in range(nt):
            seg = pos[r, i * tile:(i + 1) * tile]
            tmin[r, i], tmax[r, i] = seg.min(), seg.max()
    counts = np.zeros(N, dtype=np.int64)
    for r in range(N):
        for t in range(N):
            rk = (r + t) % N
            if causal:
                ok = tmin[rk][None, :] <= tmax[r][:, None]     # [q tiles, k tiles]
            else:
                ok = np.ones((nt, nt), dtype=bool)
            counts[r] += int(ok.sum())
    return counts


def imbalance(counts: np.ndarray) -> float:
    """max over ranks / mean over ranks."""
    return float(counts.max() / counts.mean())
