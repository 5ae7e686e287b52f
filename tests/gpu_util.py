"""Helpers for the GPU parity tests: layout the seeded inputs, read back sampled
rows of the GPU output, evaluate the oracle on the same rows, compare.

The layout of inputs and the read-back use the oracle's index maps (pure
indexing); the numbers compared come from the CUDA library on one side and the
fp64 oracle on the other.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import attention as A
from oracle import layouts as L

# Tolerances: bf16 O max-abs 2e-2 and mean-abs 2e-3, fp32 lse max-abs 1e-3.
TOL_O_MAX, TOL_O_MEAN, TOL_LSE = 2e-2, 2e-3, 1e-3


def token_map(B, S, N, layout):
    """Rank-major token index -> natural flat token (Ulysses shards are the contiguous split)."""
    return L.rank_major_map(B, S, N, "contiguous" if layout == "ulysses" else layout)


def to_layout(x: torch.Tensor, N: int, layout: str) -> torch.Tensor:
    """natural [B, S, H, D] -> the layout's input tensor [N, B, S/N, H, D] (same dtype)."""
    B, S, H, D = x.shape
    m = torch.from_numpy(token_map(B, S, N, layout))
    return x.reshape(B * S, H, D)[m].reshape(N, B, S // N, H, D).contiguous()


def from_layout(y: torch.Tensor, N: int, layout: str) -> torch.Tensor:
    """The layout's tensor [N, B, S/N, H, D] -> natural [B, S, H, D] (inverse of to_layout)."""
    N_, B, T, H, D = y.shape
    S = N * T
    m = torch.from_numpy(token_map(B, S, N, layout)).to(y.device)
    nat = torch.empty(B * S, H, D, dtype=y.dtype, device=y.device)
    nat[m] = y.reshape(B * S, H, D)
    return nat.reshape(B, S, H, D)


def gather_rows(o_layout: torch.Tensor, B, S, H, N, layout, rows: np.ndarray) -> np.ndarray:
    """Rows (b, h, i) of a layout-shaped output, as fp64 numpy [n, D]."""
    D = o_layout.shape[-1]
    m = token_map(B, S, N, layout)
    inv = np.empty_like(m)
    inv[m] = np.arange(m.size)
    flat = inv[rows[:, 0] * S + rows[:, 2]]
    idx = torch.from_numpy(flat).to(o_layout.device)
    hh = torch.from_numpy(rows[:, 1]).to(o_layout.device)
    sel = o_layout.reshape(-1, H, D)[idx, hh]
    return sel.to(torch.float64).cpu().numpy()


def oracle_rows(q, k, v, rows, causal, scale=None):
    """Oracle O [n, D] and lse [n] at natural rows (b, h, i); inputs bf16 natural (CPU)."""
    f = lambda t: t.float().numpy()        # bf16 -> fp32 is exact
    return A.attention_rows(f(q), f(k), f(v), rows, causal=causal, scale=scale)


def errors(o_gpu: np.ndarray, o_ref: np.ndarray, lse_gpu: np.ndarray, lse_ref: np.ndarray):
    d = np.abs(o_gpu - o_ref)
    return {"o_max": float(d.max()), "o_mean": float(d.mean()),
            "lse_max": float(np.abs(lse_gpu - lse_ref).max())}


def assert_within(err: dict, what: str = ""):
    assert np.isfinite(err["o_max"]) and np.isfinite(err["lse_max"]), (what, err)
    assert err["o_max"] <= TOL_O_MAX, (what, err)
    assert err["o_mean"] <= TOL_O_MEAN, (what, err)
    assert err["lse_max"] <= TOL_LSE, (what, err)
