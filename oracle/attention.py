"""Softmax attention, its per-chunk partials and their merge, in fp64 on the CPU.

Test infrastructure only (see the package docstring).

Sources on the pages:
  * "Tensor并行与算子拆分" (aiknowledge.cn), section "注意力的并行化优化"
    (parallel attention): scores are Q K^T / sqrt(d_k); masked positions are
    filled with -inf; weights are the softmax over keys; the output is the
    weights times V.
  * "序列与上下文并行" (ai-infra-wiki), section "上下文并行：注意力本身切分"
    (context parallelism): each rank holds its own Q/K/V block, K/V blocks are
    passed around a ring, each rank computes its Q against every K/V block and
    the partial results are merged incrementally by online softmax, so the
    merged result is full softmax attention.
  * Same page, section "工程实践" (practice): positions are global positions
    under context parallelism.

Readings where the pages are silent:
  * the causal mask keeps key j for query i iff pos(j) <= pos(i) (diagonal
    kept), in global positions;
  * lse is the natural logarithm of the sum of exp of the *scaled* scores;
  * the partial of a row with no allowed key is (O = 0, lse = -inf), and the
    merge of only such partials is (0, -inf);
  * the merge of partials (O_t, lse_t) is lse = M + ln sum_t exp(lse_t - M)
    with M = max_t lse_t, and O = sum_t exp(lse_t - lse) O_t.

Tensor conventions: natural layout [B, S, H, D] for Q/K/V/O (batch, token, head,
head dim), lse as [B, H, S]. All arithmetic in float64.
"""
from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence

import numpy as np

NEG_INF = -np.inf


def default_scale(D: int) -> float:
    """1/sqrt(D), the score scale of the parallel-attention section."""
    return 1.0 / math.sqrt(D)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, *, causal: bool,
              scale: Optional[float] = None,
              q_pos: Optional[np.ndarray] = None,
              k_pos: Optional[np.ndarray] = None):
    """Full softmax attention with per-row logsumexp (matrix form).

    q: [B, Sq, H, D]; k, v: [B, Sk, H, D] (float64). ``q_pos``/``k_pos`` are the
    global positions of the query/key tokens (default 0..S-1); the causal mask
    keeps key j for query i iff k_pos[j] <= q_pos[i].

    Returns (O [B, Sq, H, D], lse [B, H, Sq]); a row with no allowed key gets
    O = 0 and lse = -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Sq, H, D = q.shape
    Sk = k.shape[1]
    if scale is None:
        scale = default_scale(D)
    qp = np.arange(Sq) if q_pos is None else np.asarray(q_pos)
    kp = np.arange(Sk) if k_pos is None else np.asarray(k_pos)

    # scores s[b, h, i, j] = scale * <q_i, k_j>
    s = np.einsum("bihd,bjhd->bhij", q, k) * scale
    if causal:
        allowed = kp[None, :] <= qp[:, None]          # [Sq, Sk]
        s = np.where(allowed[None, None], s, NEG_INF)
    m = s.max(axis=-1, keepdims=True)                 # row max
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    e = np.exp(s - m_safe)                            # exp(-inf) = 0 on masked entries
    z = e.sum(axis=-1, keepdims=True)
    with np.errstate(divide="ignore"):
        lse = np.where(empty, NEG_INF, m_safe + np.log(z))
    w = np.where(empty, 0.0, e / np.where(z == 0, 1.0, z))   # softmax weights
    o = np.einsum("bhij,bjhd->bihd", w, v)
    return o, lse[..., 0]


def attention_rowloop(q, k, v, *, causal: bool, scale: Optional[float] = None):
    """Brute-force attention: one query row at a time, scalar loops over keys.

    Independent of :func:`attention` (no einsum, no masking array); used to pin
    it on tiny inputs.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, S, H, D = q.shape
    Sk = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    o = np.zeros((B, S, H, D))
    lse = np.full((B, H, S), NEG_INF)
    for b in range(B):
        for h in range(H):
            for i in range(S):
                keys = [j for j in range(Sk) if (not causal or j <= i)]
                if not keys:
                    continue
                scores = []
                for j in keys:
                    acc = 0.0
                    for d in range(D):
                        acc += q[b, i, h, d] * k[b, j, h, d]
                    scores.append(acc * scale)
                mx = max(scores)
                ex = [math.exp(x - mx) for x in scores]
                tot = math.fsum(ex)
                lse[b, h, i] = mx + math.log(tot)
                for jj, j in enumerate(keys):
                    o[b, i, h, :] += (ex[jj] / tot) * v[b, j, h, :]
    return o, lse


def attention_rows(q, k, v, rows: np.ndarray, *, causal: bool,
                   scale: Optional[float] = None):
    """Attention for selected query rows only (natural positions).

    rows: int64 [n, 3] of (b, h, i). Returns (O [n, D], lse [n]). Rows are
    grouped by (b, h) so the cost is n x S x D per group, not S^2.
    """
    B, S, H, D = q.shape
    if scale is None:
        scale = default_scale(D)
    rows = np.asarray(rows, dtype=np.int64)
    o = np.zeros((rows.shape[0], D))
    lse = np.zeros(rows.shape[0])
    keys = rows[:, 0] * H + rows[:, 1]
    order = np.argsort(keys, kind="stable")
    bounds = np.flatnonzero(np.diff(keys[order])) + 1
    for grp in np.split(order, bounds):
        if grp.size == 0:
            continue
        b, h = int(rows[grp[0], 0]), int(rows[grp[0], 1])
        ii = rows[grp, 2]
        qs = np.asarray(q[b, ii, h, :], dtype=np.float64)          # [n, D]
        ks = np.asarray(k[b, :, h, :], dtype=np.float64)           # [S, D]
        vs = np.asarray(v[b, :, h, :], dtype=np.float64)
        s = (qs @ ks.T) * scale                                    # [n, S]
        if causal:
            s = np.where(np.arange(ks.shape[0])[None, :] <= ii[:, None], s, NEG_INF)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        z = e.sum(axis=1, keepdims=True)
        lse[grp] = (m + np.log(z))[:, 0]
        o[grp] = (e / z) @ vs
    return o, lse


def partial(q_rows, q_pos, k_chunk, v_chunk, k_pos, *, causal: bool, scale: float):
    """Partial result of query rows against one key/value chunk.

    q_rows: [n, D]; k_chunk, v_chunk: [m, D]; q_pos [n], k_pos [m] global
    positions. Returns (O_t [n, D], lse_t [n]) where O_t is the softmax-weighted
    mean of V over the allowed keys of the chunk and lse_t the logsumexp of
    their scaled scores; rows with no allowed key give (0, -inf). This is what
    one ring step of the context-parallel section computes for one rank.
    """
    q_rows = np.asarray(q_rows, dtype=np.float64)
    k_chunk = np.asarray(k_chunk, dtype=np.float64)
    v_chunk = np.asarray(v_chunk, dtype=np.float64)
    n, D = q_rows.shape
    o = np.zeros((n, D))
    lse = np.full(n, NEG_INF)
    if k_chunk.shape[0] == 0:
        return o, lse
    s = (q_rows @ k_chunk.T) * scale
    if causal:
        s = np.where(np.asarray(k_pos)[None, :] <= np.asarray(q_pos)[:, None], s, NEG_INF)
    m = s.max(axis=1)
    ok = np.isfinite(m)
    if ok.any():
        e = np.exp(s[ok] - m[ok, None])
        z = e.sum(axis=1)
        lse[ok] = m[ok] + np.log(z)
        o[ok] = (e / z[:, None]) @ v_chunk
    return o, lse


def merge(parts: Sequence[tuple]):
    """Merge partials [(O_t [n, D], lse_t [n]), ...] into (O [n, D], lse [n]).

    lse = M + ln sum_t exp(lse_t - M) with M = max_t lse_t; O = sum_t
    exp(lse_t - lse) O_t. Partials with lse_t = -inf contribute nothing; rows
    whose partials are all -inf give (0, -inf).
    """
    os_ = np.stack([np.asarray(p[0], dtype=np.float64) for p in parts])   # [T, n, D]
    ls = np.stack([np.asarray(p[1], dtype=np.float64) for p in parts])    # [T, n]
    M = ls.max(axis=0)
    ok = np.isfinite(M)
    Ms = np.where(ok, M, 0.0)
    w = np.exp(ls - Ms[None])                     # 0 where lse_t = -inf
    tot = w.sum(axis=0)
    lse = np.where(ok, Ms + np.log(np.where(ok, tot, 1.0)), NEG_INF)
    coef = np.where(ok[None], w / np.where(ok, tot, 1.0)[None], 0.0)
    o = np.einsum("tn,tnd->nd", coef, os_)
    return o, lse


def merge_sequential(parts: Iterable[tuple]):
    """Merge partials one at a time, in the given (ring) order.

    The incremental form of the context-parallel section: a running
    (O, lse) pair is combined with each new partial as it arrives. Must equal
    :func:`merge` of the whole list.
    """
    run_o, run_l = None, None
    for o_t, l_t in parts:
        if run_o is None:
            run_o = np.array(o_t, dtype=np.float64)
            run_l = np.array(l_t, dtype=np.float64)
            continue
        run_o, run_l = merge([(run_o, run_l), (o_t, l_t)])
    return run_o, run_l


def ring_partials(q, k, v, layout_map, N: int, *, causal: bool, scale=None):
    """Per-rank, per-ring-step partials of the context-parallel method.

    q, k, v: natural [B, S, H, D]. ``layout_map`` is the rank-major token map of
    :mod:`oracle.layouts` (entry (r*B + b)*T + tl -> natural flat token
    b*S + pos). Rank r at ring step t uses the K/V block of rank (r + t) mod N
    (the visiting order of the context-parallel section). Returns
    parts[r][t] = (O_t [B, T, H, D], lse_t [B, H, T]) in rank r's local order.
    """
    B, S, H, D = q.shape
    T = S // N
    if scale is None:
        scale = default_scale(D)
    pos = (np.asarray(layout_map) % S).reshape(N, B, T)
    flat = lambda x: np.asarray(x, dtype=np.float64).reshape(B * S, H, D)
    qf, kf, vf = flat(q), flat(k), flat(v)
    idx = np.asarray(layout_map).reshape(N, B, T)
    out = []
    for r in range(N):
        steps = []
        for t in range(N):
            rk = (r + t) % N
            o_t = np.zeros((B, T, H, D))
            l_t = np.zeros((B, H, T))
            for b in range(B):
                qi, ki = idx[r, b], idx[rk, b]
                for h in range(H):
                    oo, ll = partial(qf[qi, h], pos[r, b], kf[ki, h], vf[ki, h],
                                     pos[rk, b], causal=causal, scale=scale)
                    o_t[b, :, h] = oo
                    l_t[b, h] = ll
            steps.append((o_t, l_t))
        out.append(steps)
    return out
