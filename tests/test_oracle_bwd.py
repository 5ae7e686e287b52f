"""Pins of the backward oracle (oracle/attention_bwd.py) against things other than
its own formulas: fp64 autograd of a plainly written attention (library), the
directional derivative of the pinned forward by central differences (calculus),
invariants and closed forms. Planted mistakes must each fail at least one pin."""
import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import attention_bwd as AB


def _rand(B, S, H, D, seed):
    g = np.random.default_rng(seed)
    return [g.standard_normal((B, S, H, D)) for _ in range(4)]


def pin_autograd(fn, causal):
    B, S, H, D = 2, 9, 2, 8
    q, k, v, do = _rand(B, S, H, D, 11 + causal)
    t = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v)]
    # attention written with torch ops only: [B, H, S, D] views
    Q, K, V = (x.permute(0, 2, 1, 3) for x in t)
    sc = Q @ K.transpose(-1, -2) / math.sqrt(D)
    if causal:
        sc = sc.masked_fill(torch.ones(S, S, dtype=torch.bool).triu(1), float("-inf"))
    out = torch.softmax(sc, dim=-1) @ V
    out.permute(0, 2, 1, 3).backward(torch.tensor(do))
    dq, dk, dv = fn(q, k, v, do, causal)
    for got, x in zip((dq, dk, dv), t):
        np.testing.assert_allclose(got, x.grad.numpy(), rtol=0, atol=1e-10)


def pin_directional_derivative(fn, causal):
    # <dX, E> = d/de sum(attention(X + e E) * dO) at e = 0, central differences on
    # the (separately pinned) forward oracle.
    B, S, H, D = 1, 12, 2, 8
    q, k, v, do = _rand(B, S, H, D, 21 + causal)
    dq, dk, dv = fn(q, k, v, do, causal)
    rng = np.random.default_rng(5)
    eps = 1e-5
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        E = rng.standard_normal(q.shape)
        args_p = [q, k, v]
        args_m = [q, k, v]
        args_p = [x + eps * E if i == which else x for i, x in enumerate(args_p)]
        args_m = [x - eps * E if i == which else x for i, x in enumerate(args_m)]
        lp = np.sum(A.attention(*args_p, causal=causal)[0] * do)
        lm = np.sum(A.attention(*args_m, causal=causal)[0] * do)
        fd = (lp - lm) / (2 * eps)
        assert abs(fd - np.sum(grad * E)) < 1e-7 * max(1.0, abs(fd)), (which, fd, np.sum(grad * E))


def pin_dk_sums_to_zero(fn, causal):
    # sum_j dS_ij = 0 for every query row, so sum over keys of dK is 0 per (b, h).
    q, k, v, do = _rand(2, 16, 3, 8, 31)
    _, dk, _ = fn(q, k, v, do, causal)
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-11)


def pin_first_causal_row(fn):
    # Query 0 sees only key 0: P = 1, dS = 0, so dQ[0] = 0; and with Q = 0 the
    # weights are uniform, so dV[j] = sum_{i >= j} dO[i] / (i + 1).
    q, k, v, do = _rand(1, 10, 1, 8, 41)
    dq, _, _ = fn(q, k, v, do, True)
    np.testing.assert_allclose(dq[0, 0], 0.0, atol=1e-12)
    _, _, dv = fn(np.zeros_like(q), k, v, do, True)
    S = q.shape[1]
    ref = np.stack([sum(do[0, i, 0] / (i + 1) for i in range(j, S)) for j in range(S)])
    np.testing.assert_allclose(dv[0, :, 0], ref, atol=1e-12)


def oracle(q, k, v, do, causal):
    dq, dk, dv, _, _ = AB.attention_bwd(q, k, v, do, causal=causal, block=4)
    return dq, dk, dv


def checks(fn):
    return [lambda: pin_autograd(fn, False), lambda: pin_autograd(fn, True),
            lambda: pin_directional_derivative(fn, False), lambda: pin_directional_derivative(fn, True),
            lambda: pin_dk_sums_to_zero(fn, True), lambda: pin_first_causal_row(fn)]


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_matches_autograd(causal):
    pin_autograd(oracle, causal)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_is_the_forward_derivative(causal):
    pin_directional_derivative(oracle, causal)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_dk_sums_to_zero(causal):
    pin_dk_sums_to_zero(oracle, causal)


def test_bwd_closed_forms():
    pin_first_causal_row(oracle)


def test_bwd_forward_outputs_match_forward_oracle():
    q, k, v, do = _rand(1, 20, 2, 8, 51)
    _, _, _, o, lse = AB.attention_bwd(q, k, v, do, causal=True, block=7)
    o_ref, lse_ref = A.attention(q, k, v, causal=True)
    np.testing.assert_allclose(o, o_ref, atol=1e-13)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-13)


def _mut(transform):
    def fn(q, k, v, do, causal):
        return transform(q, k, v, do, causal)
    return fn


def _no_D(q, k, v, do, causal):
    # dS = P * dP (the - D term dropped)
    B, S, H, D = q.shape
    dq, dk, dv = [np.zeros_like(q) for _ in range(3)]
    for b in range(B):
        for h in range(H):
            sc = q[b, :, h] @ k[b, :, h].T / math.sqrt(D)
            if causal:
                sc[np.triu(np.ones((S, S), bool), 1)] = -np.inf
            P = np.exp(sc - sc.max(1, keepdims=True))
            P /= P.sum(1, keepdims=True)
            dv[b, :, h] = P.T @ do[b, :, h]
            dS = P * (do[b, :, h] @ v[b, :, h].T)
            dq[b, :, h] = dS @ k[b, :, h] / math.sqrt(D)
            dk[b, :, h] = dS.T @ q[b, :, h] / math.sqrt(D)
    return dq, dk, dv


MUTANTS = {
    "minus_D_dropped": _no_D,
    "dq_scale_missing": _mut(lambda q, k, v, do, c: (lambda r: (r[0] * math.sqrt(q.shape[-1]), r[1], r[2]))(
        oracle(q, k, v, do, c))),
    "dk_dv_swapped": _mut(lambda q, k, v, do, c: (lambda r: (r[0], r[2], r[1]))(oracle(q, k, v, do, c))),
    "mask_ignored": _mut(lambda q, k, v, do, c: oracle(q, k, v, do, False)),
    "do_transposed_heads": _mut(lambda q, k, v, do, c: oracle(q, k, v, do[:, :, ::-1], c)),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_bwd_mutant_is_caught(name):
    fn = MUTANTS[name]

    def _fails(check):
        try:
            check()
        except AssertionError:
            return True
        return False
    assert any(_fails(c) for c in checks(fn)), name
