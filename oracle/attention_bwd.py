"""Gradients of softmax attention (the backward pass), fp64 on the CPU.

Test infrastructure only (see the package docstring).

The pages are about training long-context models (page "序列与上下文并行",
opening and section "长上下文的显存墙": activations grow with the sequence) but
print no backward pass. The method's forward is plain softmax attention (page
"Tensor并行与算子拆分", section "注意力的并行化优化": scores Q K^T / sqrt(d),
masked entries -inf, softmax over keys, weights times V), so its backward is
the derivative of that definition — the gradients of L = sum(O * dO) with
respect to Q, K and V for an upstream gradient dO — and this module writes the
chain rule out, per (batch, head), with the row logsumexp of the forward:

    P   = exp(scale * Q K^T - lse)          (masked entries 0)
    dV  = P^T dO
    dP  = dO V^T
    Dr  = rowsum(dO * O)                    (= rowsum(P * dP))
    dS  = P * (dP - Dr)
    dQ  = scale * dS K
    dK  = scale * dS^T Q

Positions are global (causal: key j is kept for query i iff pos(j) <= pos(i)),
as in the forward. Tensors are natural [B, S, H, D]; all arithmetic float64.
Query rows are processed in blocks so one head of a 32k sequence fits in memory.
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np


def attention_bwd(q, k, v, do, *, causal: bool, scale: Optional[float] = None,
                  heads=None, block: int = 512):
    """Returns (dq, dk, dv, o, lse) in fp64; dq/dk/dv/o [B, S, H, D], lse [B, H, S].

    heads: optional list of head indices to compute (others are left zero / nan-free
    zeros), for full-size checks of a few heads.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    B, S, H, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    o = np.zeros_like(q)
    lse = np.zeros((B, H, S))
    pos = np.arange(S)
    for b in range(B):
        for h in (range(H) if heads is None else heads):
            Q, K, V, G = q[b, :, h], k[b, :, h], v[b, :, h], do[b, :, h]
            # forward pass of the block rows: lse and O
            for s0 in range(0, S, block):
                s1 = min(S, s0 + block)
                sc = scale * (Q[s0:s1] @ K.T)
                if causal:
                    sc[pos[None, :] > pos[s0:s1, None]] = -np.inf
                m = sc.max(axis=1)
                p = np.exp(sc - m[:, None])
                l = p.sum(axis=1)
                lse[b, h, s0:s1] = m + np.log(l)
                o[b, s0:s1, h] = (p / l[:, None]) @ V
            # backward
            for s0 in range(0, S, block):
                s1 = min(S, s0 + block)
                sc = scale * (Q[s0:s1] @ K.T)
                if causal:
                    sc[pos[None, :] > pos[s0:s1, None]] = -np.inf
                P = np.exp(sc - lse[b, h, s0:s1, None])
                dv[b, :, h] += P.T @ G[s0:s1]
                dP = G[s0:s1] @ V.T
                Dr = np.sum(G[s0:s1] * o[b, s0:s1, h], axis=1)
                dS = P * (dP - Dr[:, None])
                dq[b, s0:s1, h] = scale * (dS @ K)
                dk[b, :, h] += scale * (dS.T @ Q[s0:s1])
    return dq, dk, dv, o, lse
