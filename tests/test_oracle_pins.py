"""The CPU oracle pinned against library special cases, closed forms and invariants."""
import math

import numpy as np
import pytest

from oracle import attention as A
from oracle import layouts as L
from tests import pins


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_sdpa(causal):
    pins.pin_sdpa(A.attention, causal)


@pytest.mark.parametrize("causal", [False, True])
def test_matrix_equals_rowloop(causal):
    pins.pin_rowloop(A.attention, A.attention_rowloop, causal)


def test_single_key_closed_form():
    pins.pin_single_key(A.attention)
    pins.pin_causal_first_row(A.attention)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_closed_form(causal):
    pins.pin_zero_query(A.attention, causal)


@pytest.mark.parametrize("causal", [False, True])
def test_weights_sum_to_one(causal):
    pins.pin_weights_sum_to_one(A.attention, causal)


@pytest.mark.parametrize("causal", [False, True])
def test_merge_all_orders(causal):
    pins.pin_merge_all_orders(A.partial, A.merge, causal=causal)
    pins.pin_merge_all_orders(A.partial, A.merge_sequential, causal=causal)


def test_merge_empty_partials():
    pins.pin_merge_empty(A.merge)


def test_rows_equal_full():
    rng = np.random.default_rng(3)
    q, k, v = (rng.standard_normal((2, 40, 3, 8)) for _ in range(3))
    o, l = A.attention(q, k, v, causal=True)
    rows = np.array([[0, 0, 0], [1, 2, 39], [0, 1, 17], [1, 0, 5]])
    o2, l2 = A.attention_rows(q, k, v, rows, causal=True)
    for n, (b, h, i) in enumerate(rows):
        np.testing.assert_allclose(o2[n], o[b, i, h], atol=1e-12)
        np.testing.assert_allclose(l2[n], l[b, h, i], atol=1e-12)


@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_partials_merge_to_full(layout, causal):
    """Per-rank ring partials merged in ring order equal full attention."""
    B, S, H, D, N = 2, 32, 2, 4, 4
    rng = np.random.default_rng(7)
    q, k, v = (rng.standard_normal((B, S, H, D)) for _ in range(3))
    o_ref, l_ref = A.attention(q, k, v, causal=causal)
    m = L.rank_major_map(B, S, N, layout)
    parts = A.ring_partials(q, k, v, m, N, causal=causal)
    T = S // N
    o_rm = np.zeros((N, B, T, H, D))
    for r in range(N):
        for b in range(B):
            for h in range(H):
                o, l = A.merge_sequential([(p[0][b, :, h], p[1][b, h]) for p in parts[r]])
                o_rm[r, b, :, h] = o
                pos = m.reshape(N, B, T)[r, b] % S
                np.testing.assert_allclose(l, l_ref[b, h, pos], atol=1e-12)
    np.testing.assert_allclose(L.from_rank_major(o_rm, layout), o_ref, atol=1e-12)


def test_zigzag_equals_contiguous_after_unpermute():
    """Attention on the zigzag rank-major token order, with global positions, un-permuted,
    equals attention on the contiguous order un-permuted (and the natural result)."""
    B, S, H, D, N = 1, 64, 2, 8, 4
    rng = np.random.default_rng(11)
    q, k, v = (rng.standard_normal((B, S, H, D)) for _ in range(3))
    outs = []
    for layout in ("contiguous", "zigzag"):
        m = L.rank_major_map(B, S, N, layout)
        pos = m % S
        qr, kr, vr = (x.reshape(B * S, H, D)[m].reshape(1, S, H, D) for x in (q, k, v))
        o, lse = A.attention(qr, kr, vr, causal=True, q_pos=pos, k_pos=pos)
        outs.append(L.from_rank_major(o.reshape(N, B, S // N, H, D), layout))
    np.testing.assert_allclose(outs[0], outs[1], rtol=0, atol=1e-12)
    np.testing.assert_allclose(outs[0], A.attention(q, k, v, causal=True)[0], rtol=0, atol=1e-12)


def test_scale_default_is_inverse_sqrt_d():
    assert A.default_scale(64) == 1 / 8
    assert A.default_scale(128) == 1 / math.sqrt(128)
