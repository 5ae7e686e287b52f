"""Pins of the sequence-parallel LayerNorm/dropout oracle (oracle/sp_norm.py):
torch's layer_norm (library), the pages' own check that per-shard LayerNorm
concatenates to LayerNorm of the whole sequence, reduce-scatter of a
row-parallel product against the full matrix product (library), closed forms.
Planted mistakes must each fail a pin."""
import numpy as np
import pytest
import torch

from oracle import sp_norm as SP


def _x(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def pin_layer_norm_library(ln):
    x, g, b = _x((7, 64), 1), _x(64, 2), _x(64, 3)
    ref = torch.nn.functional.layer_norm(torch.tensor(x), (64,), torch.tensor(g), torch.tensor(b), eps=1e-5)
    np.testing.assert_allclose(ln(x, g, b), ref.numpy(), atol=1e-12)


def pin_shards_concatenate_to_full(ln):
    # The 5688vip.com page's verification: LayerNorm of each rank's sequence
    # shard, concatenated, equals LayerNorm of the whole sequence.
    x, g, b = _x((12, 8), 42), _x(8, 43), _x(8, 44)
    N = 3
    shards = np.split(x, N, axis=0)
    cat = np.concatenate([ln(s, g, b) for s in shards], axis=0)
    np.testing.assert_allclose(cat, ln(x, g, b), atol=1e-12)
    # and the normalised rows have mean 0 and population variance ~1 before gamma/beta
    y = ln(x, np.ones(8), np.zeros(8))
    np.testing.assert_allclose(y.mean(axis=-1), 0.0, atol=1e-12)
    np.testing.assert_allclose(y.var(axis=-1), 1.0, rtol=1e-3)


def pin_reduce_scatter_is_row_parallel_product(rs):
    # Tensor parallelism of a row-parallel linear: rank r holds columns K_r of X and
    # rows K_r of W; its partial X[:, K_r] W[K_r, :] summed over ranks is X W.
    S, K, H, N = 16, 24, 8, 4
    X, W = _x((S, K), 5), _x((K, H), 6)
    parts = np.stack([X[:, r * K // N:(r + 1) * K // N] @ W[r * K // N:(r + 1) * K // N] for r in range(N)])
    shards = rs(parts, N)
    np.testing.assert_allclose(SP.all_gather(shards), torch.tensor(X).matmul(torch.tensor(W)).numpy(), atol=1e-12)
    assert shards.shape == (N, S // N, H)


def pin_fused_closed_forms(fused):
    S, H, N, p = 8, 32, 2, 0.25
    parts, res, g, b = _x((N, S, H), 7), _x((S, H), 8), _x(H, 9), _x(H, 10)
    keep_all = np.ones((S, H), bool)
    z, y = fused(parts, keep_all, p, res, g, b)
    np.testing.assert_allclose(z, parts.sum(0) / (1 - p) + res, atol=1e-12)
    keep_none = np.zeros((S, H), bool)
    z, y = fused(parts, keep_none, p, res, g, b)
    np.testing.assert_allclose(z, res, atol=1e-12)
    ref = torch.nn.functional.layer_norm(torch.tensor(res), (H,), torch.tensor(g), torch.tensor(b), eps=1e-5)
    np.testing.assert_allclose(y, ref.numpy(), atol=1e-12)


def test_layer_norm_library():
    pin_layer_norm_library(SP.layer_norm)


def test_shards_concatenate_to_full():
    pin_shards_concatenate_to_full(SP.layer_norm)


def test_reduce_scatter():
    pin_reduce_scatter_is_row_parallel_product(SP.reduce_scatter)


def test_fused_closed_forms():
    pin_fused_closed_forms(SP.rs_dropout_add_ln)


def _ln_unbiased(x, g, b, eps=1e-5):
    x = np.asarray(x, np.float64)
    return (x - x.mean(-1, keepdims=True)) / np.sqrt(x.var(-1, ddof=1, keepdims=True) + eps) * g + b


def _ln_eps_outside(x, g, b, eps=1e-5):
    x = np.asarray(x, np.float64)
    return (x - x.mean(-1, keepdims=True)) / (np.sqrt(x.var(-1, keepdims=True)) + eps) * g + b


def _ln_full_sequence_stats(x, g, b, eps=1e-5):
    # statistics over the sequence instead of the hidden dimension
    x = np.asarray(x, np.float64)
    return (x - x.mean(0, keepdims=True)) / np.sqrt(x.var(0, keepdims=True) + eps) * g + b


def _rs_first_partial_only(parts, N):
    return np.stack(np.split(np.asarray(parts, np.float64)[0], N, axis=0))


def _fused_no_rescale(parts, keep, p, res, g, b, eps=1e-5):
    z = np.where(keep, np.asarray(parts, np.float64).sum(0), 0.0) + res
    return z, SP.layer_norm(z, g, b, eps)


MUTANTS = {
    "ln_unbiased_variance": ("ln", _ln_unbiased),
    "ln_eps_outside_sqrt": ("ln", _ln_eps_outside),
    "ln_over_sequence": ("ln", _ln_full_sequence_stats),
    "rs_drops_partials": ("rs", _rs_first_partial_only),
    "dropout_not_rescaled": ("fused", _fused_no_rescale),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_sp_mutant_is_caught(name):
    kind, fn = MUTANTS[name]
    checks = {"ln": [lambda: pin_layer_norm_library(fn), lambda: pin_shards_concatenate_to_full(fn)],
              "rs": [lambda: pin_reduce_scatter_is_row_parallel_product(fn)],
              "fused": [lambda: pin_fused_closed_forms(fn)]}[kind]

    def _fails(c):
        try:
            c()
        except AssertionError:
            return True
        return False
    assert any(_fails(c) for c in checks), name
