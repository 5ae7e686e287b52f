"""Megatron-style sequence parallelism around LayerNorm/Dropout — test
infrastructure only.

Sources on the pages:
  * "序列并行：超长序列训练" (guijiagi.com), the MegatronSP example: LayerNorm is
    computed on each rank's sequence shard with no communication (it is per
    token); after the tensor-parallel region a reduce-scatter along the sequence
    returns each rank its shard of the summed result; dropout is applied locally
    and the residual is added.
  * "序列与上下文并行" (ai-infra-wiki), section "TP-SP": the tensor-parallel
    all-reduce is split into all-gather + reduce-scatter, which convert between
    the hidden-sharded and the sequence-sharded regions.
  * The 5688vip.com page, its sequence_parallel_ln_dropout function: LayerNorm
    over the hidden dimension with the population variance and eps = 1e-5,
    gamma * x_norm + beta, then dropout in training mode (keep where a uniform
    draw exceeds the drop rate, kept values divided by 1 - rate); its check that
    the per-shard results, concatenated, equal LayerNorm of the whole sequence.

Readings where the pages leave it open: the fused op after a tensor-parallel region is
    z = dropout(reduce_scatter(partials)) + residual,   y = LayerNorm(z),
with the keep mask an input (the random draw the method makes); reduce-scatter
over N ranks sums the N partial [S, ...] tensors and hands rank i its i-th
contiguous sequence chunk; all-gather concatenates the chunks in rank order.
All arithmetic float64.
"""
from __future__ import annotations

import numpy as np


def layer_norm(x, gamma, beta, eps: float = 1e-5):
    """LayerNorm over the last dimension: population variance, eps inside the sqrt."""
    x = np.asarray(x, dtype=np.float64)
    mean = x.mean(axis=-1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=-1, keepdims=True)
    return (x - mean) / np.sqrt(var + eps) * np.asarray(gamma, np.float64) + np.asarray(beta, np.float64)


def dropout(x, keep, p: float):
    """Training-mode dropout with a given keep mask: kept values / (1 - p), others 0."""
    return np.where(keep, np.asarray(x, np.float64) / (1.0 - p), 0.0)


def reduce_scatter(partials, N: int):
    """partials [N, S, ...] (one partial sum per rank) -> shards [N, S/N, ...] of their sum."""
    total = np.asarray(partials, np.float64).sum(axis=0)
    return np.stack(np.split(total, N, axis=0))


def all_gather(shards):
    """shards [N, S/N, ...] -> [S, ...], concatenated in rank order."""
    return np.concatenate(list(shards), axis=0)


def rs_dropout_add_ln(partials, keep, p, residual, gamma, beta, eps: float = 1e-5):
    """Fused step after a tensor-parallel region, on every rank's shard at once.

    partials [N, S, H] (N >= 1), keep bool [S, H] or None, residual [S, H] or None,
    gamma/beta [H] or None. Returns (z, y) as [S, H] (the shards in rank order);
    y is None without gamma.
    """
    N = np.asarray(partials).shape[0]
    z = all_gather(reduce_scatter(partials, N))
    if keep is not None:
        z = dropout(z, keep, p)
    if residual is not None:
        z = z + np.asarray(residual, np.float64)
    y = layer_norm(z, gamma, beta, eps) if gamma is not None else None
    return z, y
