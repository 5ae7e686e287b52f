"""Pin checks for the CPU oracle.

Each check takes the function under test as an argument and raises
AssertionError when it disagrees with something the pages or the mathematics
fix. ``test_oracle_pins.py`` runs them on the oracle; ``test_oracle_mutations``
runs them on deliberately broken variants of the oracle (mistakes planted on
the CPU) and requires that every variant fails at least one of them.
"""
from __future__ import annotations

import itertools
import math

import numpy as np
import torch


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def pin_sdpa(attn, causal: bool, B=2, S=24, H=3, D=8, seed=0):
    """Matches torch's scaled_dot_product_attention (fp64, CPU) and torch.logsumexp."""
    q, k, v = (_rand((B, S, H, D), seed + i) for i in range(3))
    o, lse = attn(q, k, v, causal=causal)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal)
    ref = ref.permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    scores = torch.matmul(tq, tk.transpose(-1, -2)) / math.sqrt(D)
    if causal:
        scores = scores.masked_fill(torch.ones(S, S, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(scores, dim=-1).numpy(), rtol=0, atol=1e-12)


def pin_rowloop(attn, rowloop, causal: bool, B=1, S=9, H=2, D=5, seed=10):
    """Matrix form equals the brute-force row loop to 1e-12."""
    q, k, v = (_rand((B, S, H, D), seed + i) for i in range(3))
    o1, l1 = attn(q, k, v, causal=causal)
    o2, l2 = rowloop(q, k, v, causal=causal)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def pin_single_key(attn, D=16, seed=20):
    """One key: O = V[0] and lse = scale * <q, k_0> for every query."""
    q = _rand((1, 5, 2, D), seed)
    k = _rand((1, 1, 2, D), seed + 1)
    v = _rand((1, 1, 2, D), seed + 2)
    o, lse = attn(q, k, v, causal=False)
    np.testing.assert_allclose(o, np.broadcast_to(v, o.shape), rtol=0, atol=1e-14)
    s0 = np.einsum("bihd,bhd->bhi", q, k[:, 0]) / math.sqrt(D)
    np.testing.assert_allclose(lse, s0, rtol=0, atol=1e-14)


def pin_causal_first_row(attn, S=7, D=4, seed=25):
    """Causal row 0 sees only key 0: O = V[0], lse = scale * <q_0, k_0>."""
    q, k, v = (_rand((1, S, 1, D), seed + i) for i in range(3))
    o, lse = attn(q, k, v, causal=True)
    np.testing.assert_allclose(o[0, 0, 0], v[0, 0, 0], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0, 0], q[0, 0, 0] @ k[0, 0, 0] / math.sqrt(D), atol=1e-14)


def pin_zero_query(attn, causal: bool, S=12, D=6, seed=30):
    """Q = 0: all scores 0, so lse_i = ln(#keys) and O_i = mean of the allowed V rows."""
    q = np.zeros((1, S, 2, D))
    k, v = _rand((1, S, 2, D), seed), _rand((1, S, 2, D), seed + 1)
    o, lse = attn(q, k, v, causal=causal)
    for i in range(S):
        n = i + 1 if causal else S
        np.testing.assert_allclose(lse[0, :, i], math.log(n), rtol=0, atol=1e-13)
        np.testing.assert_allclose(o[0, i], v[0, :n].mean(axis=0), rtol=0, atol=1e-13)


def pin_weights_sum_to_one(attn, causal: bool, S=10, D=4, seed=40):
    """V = 1 makes O the sum of the softmax weights: exactly 1 up to rounding."""
    q, k = _rand((2, S, 3, D), seed), _rand((2, S, 3, D), seed + 1)
    o, _ = attn(q, k, np.ones((2, S, 3, D)), causal=causal)
    assert np.abs(o - 1.0).max() < 1e-12


def pin_merge_all_orders(partial, merge, N=4, S=16, D=8, causal=True, seed=50):
    """Keys split into N chunks; merging the partials in all N! orders equals full attention."""
    from oracle.attention import attention
    q, k, v = (_rand((1, S, 1, D), seed + i) for i in range(3))
    o_ref, l_ref = attention(q, k, v, causal=causal)
    c = S // N
    pos = np.arange(S)
    parts = []
    for t in range(N):
        sl = slice(t * c, (t + 1) * c)
        parts.append(partial(q[0, :, 0], pos, k[0, sl, 0], v[0, sl, 0], pos[sl],
                             causal=causal, scale=1 / math.sqrt(D)))
    for perm in itertools.permutations(range(N)):
        o, l = merge([parts[i] for i in perm])
        np.testing.assert_allclose(o, o_ref[0, :, 0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(l, l_ref[0, 0], rtol=0, atol=1e-12)


def pin_merge_empty(merge, D=4, seed=60):
    """A (0, -inf) partial changes nothing; only-empty partials give (0, -inf)."""
    o1, l1 = _rand((3, D), seed), _rand(3, seed + 1)
    empty = (np.zeros((3, D)), np.full(3, -np.inf))
    o, l = merge([empty, (o1, l1), empty])
    np.testing.assert_allclose(o, o1, rtol=0, atol=1e-15)
    np.testing.assert_allclose(l, l1, rtol=0, atol=1e-15)
    o, l = merge([empty, empty])
    assert np.all(o == 0) and np.all(np.isneginf(l))
