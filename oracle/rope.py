"""Rotary position embedding at global positions — test infrastructure only.

Source: page "序列与上下文并行" (ai-infra-wiki), section "工程实践": under context
parallelism every rank must apply position encodings at the GLOBAL position of
each of its tokens (its segment's offset in the whole sequence), and getting
those offsets wrong is called the most common bug. The pages use RoPE there
without writing it out; their only printed position encoding is the sinusoidal
one of page "Tensor并行与算子拆分" (aiknowledge.cn), the PositionalEncoding class
of its model example: frequencies 10000^(-2i/d) on the even/odd feature pairs.

Reading, where the pages name no rotary formula: rotary embedding with that base and pairing —
feature pair (2i, 2i+1) of a head vector at global position p is rotated by the
angle p * theta_i, theta_i = base^(-2i/D):
    y[2i]   = x[2i] cos(p theta_i) - x[2i+1] sin(p theta_i)
    y[2i+1] = x[2i] sin(p theta_i) + x[2i+1] cos(p theta_i)
Computed in fp64 by that definition.
"""
from __future__ import annotations

import numpy as np


def theta(D: int, base: float = 10000.0) -> np.ndarray:
    """fp64 [D/2]: theta_i = base^(-2i/D)."""
    i = np.arange(D // 2, dtype=np.float64)
    return base ** (-2.0 * i / D)


def rope(x: np.ndarray, pos: np.ndarray, base: float = 10000.0) -> np.ndarray:
    """Rotate x [..., P, H, D] (any leading dims; P tokens) at positions pos [P].

    Returns fp64 of the same shape.
    """
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[:, None] * theta(D, base)[None, :]   # [P, D/2]
    c = np.cos(ang)[:, None, :]                                                 # [P, 1, D/2]
    s = np.sin(ang)[:, None, :]
    xe, xo = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = xe * c - xo * s
    y[..., 1::2] = xe * s + xo * c
    return y
