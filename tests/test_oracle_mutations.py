"""Planted mistakes in the oracle (on the CPU) must each fail at least one pin.

Each mutant wraps the oracle with one plausible mistake — a wrong scale, a
transposed operand, a dropped diagonal, a dropped or sign-flipped merge term, an
off-by-one position — and the pins of ``tests/pins.py`` must catch it.
"""
import math

import numpy as np
import pytest

from oracle import attention as A
from tests import pins


def _fails(check):
    try:
        check()
    except AssertionError:
        return True
    return False


def attn_checks(fn):
    return [
        lambda: pins.pin_sdpa(fn, False),
        lambda: pins.pin_sdpa(fn, True),
        lambda: pins.pin_single_key(fn),
        lambda: pins.pin_causal_first_row(fn),
        lambda: pins.pin_zero_query(fn, True),
        lambda: pins.pin_zero_query(fn, False),
        lambda: pins.pin_weights_sum_to_one(fn, True),
    ]


ATTN_MUTANTS = {
    "scale_sqrt_missing": lambda q, k, v, causal: A.attention(q, k, v, causal=causal, scale=1.0),
    "scale_off_by_1pct": lambda q, k, v, causal: A.attention(
        q, k, v, causal=causal, scale=1.01 / math.sqrt(q.shape[-1])),
    "k_v_swapped": lambda q, k, v, causal: A.attention(q, v, k, causal=causal),
    "diagonal_dropped": lambda q, k, v, causal: A.attention(
        q, k, v, causal=causal, q_pos=np.arange(q.shape[1]) - 1),
    "mask_off_by_one_up": lambda q, k, v, causal: A.attention(
        q, k, v, causal=causal, q_pos=np.arange(q.shape[1]) + 1),
    "no_causal_mask": lambda q, k, v, causal: A.attention(q, k, v, causal=False),
    "lse_log2": lambda q, k, v, causal: (lambda r: (r[0], r[1] / math.log(2)))(
        A.attention(q, k, v, causal=causal)),
    "heads_mixed": lambda q, k, v, causal: A.attention(q, k[:, :, ::-1], v[:, :, ::-1], causal=causal),
}


@pytest.mark.parametrize("name", sorted(ATTN_MUTANTS))
def test_attention_mutant_is_caught(name):
    fn = ATTN_MUTANTS[name]
    assert any(_fails(c) for c in attn_checks(fn)), name


def _merge_drop_last(parts):
    return A.merge(list(parts)[:-1])


def _merge_sign_flip(parts):
    os_ = np.stack([p[0] for p in parts])
    ls = np.stack([p[1] for p in parts])
    M = ls.max(axis=0)
    w = np.exp(-(ls - M))                      # wrong sign in the weight exponent
    lse = M + np.log(w.sum(axis=0))
    return np.einsum("tn,tnd->nd", w / w.sum(axis=0), os_), lse


def _merge_unweighted(parts):
    os_ = np.stack([p[0] for p in parts])
    ls = np.stack([p[1] for p in parts])
    M = ls.max(axis=0)
    return os_.mean(axis=0), M + np.log(np.exp(ls - M).sum(axis=0))


def _merge_empty_nan(parts):
    os_ = np.stack([p[0] for p in parts])
    ls = np.stack([p[1] for p in parts])
    M = ls.max(axis=0)
    w = np.exp(ls - M)                         # -inf - -inf = nan on all-empty rows
    lse = M + np.log(w.sum(axis=0))
    return np.einsum("tn,tnd->nd", w / w.sum(axis=0), os_), lse


@pytest.mark.parametrize("fn", [_merge_drop_last, _merge_sign_flip, _merge_unweighted, _merge_empty_nan])
def test_merge_mutant_is_caught(fn):
    checks = [lambda: pins.pin_merge_all_orders(A.partial, fn),
              lambda: pins.pin_merge_empty(fn)]
    with np.errstate(all="ignore"):
        assert any(_fails(c) for c in checks)


def test_partial_mutant_is_caught():
    def partial_no_mask(qr, qp, kc, vc, kp, *, causal, scale):
        return A.partial(qr, qp, kc, vc, kp, causal=False, scale=scale)
    assert _fails(lambda: pins.pin_merge_all_orders(partial_no_mask, A.merge))
