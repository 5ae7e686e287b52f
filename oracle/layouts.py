"""Token layouts of the virtual ranks, as int64 index maps — test infrastructure only.

Sources on the pages:
  * "序列并行：超长序列训练" (guijiagi.com), the opening split diagram: rank i
    holds tokens [i*L/N, (i+1)*L/N) (contiguous sequence sharding).
  * "序列与上下文并行" (ai-infra-wiki), section "上下文并行：注意力本身切分":
    causal load imbalance is fixed by a zigzag assignment. The pages do not
    define the zigzag; the reading used here (and by the workloads) is: the
    sequence is cut into 2N chunks of C = S/(2N) tokens and rank r holds chunks
    r and 2N-1-r, in that order.
  * "序列并行：超长序列训练", the UlyssesAttention example: an all-to-all turns
    sequence shards holding every head into head groups holding the whole
    sequence. Reading: group g holds the contiguous heads
    [g*H/N, (g+1)*H/N); the inverse all-to-all maps back.

Layouts (element order, outermost first):
  natural            [B, S, H, D]
  rank-major         [N, B, T, H, D]; T = S/N local tokens per rank
  Ulysses shards     [N, B, S/N, H, D]   (= contiguous rank-major)
  Ulysses groups     [N, B, S, H/N, D]
"""
from __future__ import annotations

import numpy as np


def chunk_positions(S: int, N: int, layout: str) -> np.ndarray:
    """Global positions of each rank's local tokens: int64 [N, T]."""
    T = S // N
    pos = np.empty((N, T), dtype=np.int64)
    if layout == "contiguous":
        for r in range(N):
            pos[r] = np.arange(r * T, (r + 1) * T)
    elif layout == "zigzag":
        C = S // (2 * N)
        for r in range(N):
            pos[r, :C] = np.arange(r * C, (r + 1) * C)
            hi = 2 * N - 1 - r
            pos[r, C:] = np.arange(hi * C, (hi + 1) * C)
    else:
        raise ValueError(layout)
    return pos


def rank_major_map(B: int, S: int, N: int, layout: str) -> np.ndarray:
    """int64 [N*B*T]: entry (r*B + b)*T + tl -> natural flat token b*S + pos."""
    pos = chunk_positions(S, N, layout)           # [N, T]
    T = S // N
    out = np.empty((N, B, T), dtype=np.int64)
    for r in range(N):
        for b in range(B):
            out[r, b] = b * S + pos[r]
    return out.reshape(-1)


def to_rank_major(x: np.ndarray, N: int, layout: str) -> np.ndarray:
    """natural [B, S, H, D] -> rank-major [N, B, T, H, D] (a gather of token rows)."""
    B, S, H, D = x.shape
    m = rank_major_map(B, S, N, layout)
    return np.asarray(x).reshape(B * S, H, D)[m].reshape(N, B, S // N, H, D)


def from_rank_major(y: np.ndarray, layout: str) -> np.ndarray:
    """rank-major [N, B, T, H, D] -> natural [B, S, H, D] (the inverse scatter)."""
    N, B, T, H, D = y.shape
    S = N * T
    m = rank_major_map(B, S, N, layout)
    out = np.empty((B * S, H, D), dtype=y.dtype)
    out[m] = y.reshape(N * B * T, H, D)
    return out.reshape(B, S, H, D)


def ulysses_run_map(B: int, S: int, H: int, N: int) -> np.ndarray:
    """int64 [N*B*S]: run i of the head-group tensor <- run map[i] of the shards.

    A run is the H/N heads x D values of one (group, batch, token). Output run
    i = (g*B + b)*S + s; its source, in the shards tensor viewed as runs
    [N, B, S/N, N], is ((rho*B + b)*(S/N) + s mod (S/N))*N + g with
    rho = s div (S/N) the shard that holds token s.
    """
    Sl = S // N
    out = np.empty((N, B, S), dtype=np.int64)
    s = np.arange(S)
    rho, sl = s // Sl, s % Sl
    for g in range(N):
        for b in range(B):
            out[g, b] = ((rho * B + b) * Sl + sl) * N + g
    return out.reshape(-1)


def shards_to_groups(x: np.ndarray, N: int) -> np.ndarray:
    """Ulysses shards [N, B, S/N, H, D] -> head groups [N, B, S, H/N, D]."""
    _, B, Sl, H, D = x.shape
    S, Hg = Sl * N, H // N
    m = ulysses_run_map(B, S, H, N)
    runs = np.asarray(x).reshape(N * B * Sl * N, Hg, D)
    return runs[m].reshape(N, B, S, Hg, D)


def groups_to_shards(y: np.ndarray) -> np.ndarray:
    """Ulysses head groups [N, B, S, H/N, D] -> shards [N, B, S/N, H, D]."""
    N, B, S, Hg, D = y.shape
    H = Hg * N
    m = ulysses_run_map(B, S, H, N)
    out = np.empty((N * B * S, Hg, D), dtype=y.dtype)
    out[m] = y.reshape(N * B * S, Hg, D)
    return out.reshape(N, B, S // N, H, D)
