"""GPU parity of the backward pass (cp_attn_bwd) against the fp64 oracle.

Tolerance, from the arithmetic: dQ, dK, dV are bf16 outputs; P and dS enter the
tensor-core products as bf16 (relative rounding 2^-9 each) and Dr = rowsum(dO*O)
uses the forward's bf16 O, so dS = P (dP - Dr) carries an absolute error of about
2^-9 P |Dr| that no per-element relative bound covers where dP and Dr cancel.
The bar is therefore per tensor, normalised by its own scale: max-abs error <=
2^-6 max|ref| and mean-abs error <= 2^-7 mean|ref| (a few bf16 roundings).
"""
import numpy as np
import pytest
import torch

import context_long_sequence_cp_b200 as cp
from oracle import attention_bwd as AB
from tests import gpu_util as G
from workloads import WORKLOADS, make_dout, make_qkv, make_small

pytestmark = pytest.mark.gpu

TOL_MAX, TOL_MEAN = 2.0 ** -6, 2.0 ** -7


def run_bwd(q, k, v, do, N, layout, causal):
    B, S, H, D = q.shape
    plan = cp.Plan(B, H, S, D, N, causal, layout)
    qd, kd, vd, dod = (G.to_layout(x, N, layout).cuda() for x in (q, k, v, do))
    o, lse = cp.attn_fwd(plan, qd, kd, vd)
    dq, dk, dv = cp.attn_bwd(plan, qd, kd, vd, o, lse, dod)
    assert cp.check(plan) == 0
    plan.close()
    return [G.from_layout(x, N, layout).double().cpu().numpy() for x in (dq, dk, dv)]


def compare(got, ref, what, heads=None):
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        if heads is not None:
            g, r = g[:, :, heads], r[:, :, heads]
        err = np.abs(g - r)
        assert np.isfinite(g).all(), (what, name)
        assert err.max() <= TOL_MAX * np.abs(r).max(), (what, name, float(err.max()), float(np.abs(r).max()))
        assert err.mean() <= TOL_MEAN * np.abs(r).mean(), (what, name, float(err.mean()), float(np.abs(r).mean()))


SMALL = [
    # (B, H, S, D, N, layout, causal, seed)
    (1, 2, 256, 64, 4, "contiguous", False, 0),
    (2, 3, 1024, 64, 2, "zigzag", True, 11),
    (2, 3, 384, 128, 3, "zigzag", True, 12),     # 64-token zigzag chunks: tiles straddle chunks
    (1, 2, 800, 128, 4, "contiguous", True, 13),  # ragged tails: 200 tokens per rank
    (1, 4, 2048, 128, 4, "zigzag", True, 14),
    (1, 2, 3000, 64, 5, "zigzag", True, 15),     # D = 64, ragged 300-token chunks, walks past every ring
    (2, 2, 1400, 128, 2, "contiguous", False, 16),  # ragged non-causal: 700 tokens per rank
]


@pytest.mark.parametrize("B,H,S,D,N,layout,causal,seed", SMALL)
def test_bwd_small_shapes_all_rows(B, H, S, D, N, layout, causal, seed):
    q, k, v = make_small(B, H, S, D, seed=seed)
    do = make_dout((B, S, H, D), seed)
    got = run_bwd(q, k, v, do, N, layout, causal)
    dq, dk, dv, _, _ = AB.attention_bwd(*(x.float().numpy() for x in (q, k, v, do)), causal=causal)
    compare(got, (dq, dk, dv), f"{layout} S={S} D={D} causal={causal}")


def test_bwd_zigzag_4k_all_heads():
    w = WORKLOADS["zigzag_4k"]
    q, k, v = make_qkv(w)
    do = make_dout(q.shape, w.seed)
    got = run_bwd(q, k, v, do, w.N, w.layout, w.causal)
    dq, dk, dv, _, _ = AB.attention_bwd(*(x.float().numpy() for x in (q, k, v, do)), causal=True, block=1024)
    compare(got, (dq, dk, dv), "zigzag_4k")


def test_bwd_zigzag_32k_one_full_head():
    w = WORKLOADS["zigzag_32k"]
    q, k, v = make_qkv(w)
    do = make_dout(q.shape, w.seed)
    got = run_bwd(q, k, v, do, w.N, w.layout, w.causal)
    head = 5
    one = [x[:, :, head:head + 1].float().numpy() for x in (q, k, v, do)]
    dq, dk, dv, _, _ = AB.attention_bwd(*one, causal=True, block=1024)
    compare([g[:, :, head:head + 1] for g in got], (dq, dk, dv), "zigzag_32k head 5")


def test_bwd_is_deterministic():
    q, k, v = make_small(1, 2, 1024, 128, seed=15)
    do = make_dout(q.shape, 15)
    a = run_bwd(q, k, v, do, 4, "zigzag", True)
    b = run_bwd(q, k, v, do, 4, "zigzag", True)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
