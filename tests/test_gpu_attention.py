"""GPU parity of the fused context-parallel attention (cp_attn_fwd) against the fp64 oracle.

Small and edge shapes compare every row; the full-size workloads compare the
seeded sampled rows (4096 random rows plus chunk-edge rows).
"""
import numpy as np
import pytest
import torch

import context_long_sequence_cp_b200 as cp
from tests import gpu_util as G
from workloads import WORKLOADS, make_qkv, make_small, sample_rows

pytestmark = pytest.mark.gpu


def run_and_compare(q, k, v, N, layout, causal, rows=None, scale=0.0, what=""):
    B, S, H, D = q.shape
    plan = cp.Plan(B, H, S, D, N, causal, layout, softmax_scale=scale)
    qd, kd, vd = (G.to_layout(x, N, layout).cuda() for x in (q, k, v))
    o, lse = cp.attn_fwd(plan, qd, kd, vd)
    assert cp.check(plan) == 0
    if rows is None:
        bb, hh, ii = np.meshgrid(np.arange(B), np.arange(H), np.arange(S), indexing="ij")
        rows = np.stack([bb.ravel(), hh.ravel(), ii.ravel()], 1).astype(np.int64)
    o_gpu = G.gather_rows(o, B, S, H, N, layout, rows)
    lse_gpu = lse.cpu().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]].astype(np.float64)
    o_ref, lse_ref = G.oracle_rows(q, k, v, rows, causal, scale=scale if scale > 0 else None)
    err = G.errors(o_gpu, o_ref, lse_gpu, lse_ref)
    G.assert_within(err, what)
    plan.close()
    return o, lse, err


SMALL = [
    # (B, H, S, D, N, layout, causal, seed)
    (1, 2, 256, 64, 4, "contiguous", False, 0),     # the tiny workload's shape, 64-token chunks
    (2, 3, 1024, 64, 2, "zigzag", True, 11),        # D = 64, causal zigzag
    (2, 3, 384, 128, 3, "zigzag", True, 12),        # 64-token zigzag chunks: tiles straddle chunks
    (1, 2, 800, 128, 4, "contiguous", True, 13),    # ragged tail: 200 tokens per rank
    (1, 2, 1000, 64, 5, "zigzag", True, 14),        # ragged, 100-token chunks
    (2, 2, 600, 128, 3, "contiguous", False, 15),   # ragged non-causal
    (1, 4, 700, 128, 1, "contiguous", True, 16),    # one rank: plain causal attention
    (1, 1, 64, 128, 1, "contiguous", False, 17),    # shorter than one tile
    (2, 8, 512, 128, 4, "ulysses", False, 18),      # Ulysses head groups of 2
    (1, 2, 2048, 128, 2, "zigzag", True, 19),       # several full tiles per chunk
]


@pytest.mark.parametrize("B,H,S,D,N,layout,causal,seed", SMALL)
def test_small_shapes_all_rows(B, H, S, D, N, layout, causal, seed):
    q, k, v = make_small(B, H, S, D, seed)
    run_and_compare(q, k, v, N, layout, causal, what=f"{B},{H},{S},{D},{N},{layout},{causal}")


def test_softmax_scale_override():
    q, k, v = make_small(1, 2, 512, 128, 21)
    run_and_compare(q, k, v, 2, "zigzag", True, scale=0.3, what="scale=0.3")


def test_tiny_workload():
    w = WORKLOADS["tiny"]
    q, k, v = make_qkv(w)
    run_and_compare(q, k, v, w.N, w.layout, w.causal, what=w.name)


def test_zigzag_4k_workload_all_rows():
    w = WORKLOADS["zigzag_4k"]
    q, k, v = make_qkv(w)
    run_and_compare(q, k, v, w.N, w.layout, w.causal, what=w.name)


def test_zigzag_32k_workload_sampled():
    w = WORKLOADS["zigzag_32k"]
    q, k, v = make_qkv(w)
    run_and_compare(q, k, v, w.N, w.layout, w.causal, rows=sample_rows(w), what=w.name)


def test_long_128k_contiguous_and_zigzag():
    """Both ring orders match the oracle and agree with each other on every row."""
    w = WORKLOADS["long_128k"]
    q, k, v = make_qkv(w)
    rows = sample_rows(w)
    outs = []
    for layout in (w.layout, w.alt_layout):
        o, lse, _ = run_and_compare(q, k, v, w.N, layout, w.causal, rows=rows, what=f"{w.name}/{layout}")
        # back to natural order for the cross-check
        m = torch.from_numpy(G.token_map(w.B, w.S, w.N, layout)).cuda()
        nat = torch.empty(w.B * w.S, w.H, w.D, dtype=o.dtype, device=o.device)
        nat[m] = o.reshape(-1, w.H, w.D)
        outs.append((nat, lse))
        del o
    d = (outs[0][0].float() - outs[1][0].float()).abs()
    assert d.max().item() <= G.TOL_O_MAX and d.mean().item() <= G.TOL_O_MEAN
    assert (outs[0][1] - outs[1][1]).abs().max().item() <= G.TOL_LSE


def test_ulysses_16k_workload_sampled():
    w = WORKLOADS["ulysses_16k"]
    q, k, v = make_qkv(w)
    run_and_compare(q, k, v, w.N, w.layout, w.causal, rows=sample_rows(w), what=w.name)


def test_repeated_calls_are_identical():
    """The same call twice gives bit-identical results (no state carried between calls)."""
    q, k, v = make_small(1, 4, 2048, 128, 31)
    plan = cp.Plan(1, 4, 2048, 128, 4, True, "zigzag")
    qd, kd, vd = (G.to_layout(x, 4, "zigzag").cuda() for x in (q, k, v))
    o1, l1 = cp.attn_fwd(plan, qd, kd, vd)
    o2, l2 = cp.attn_fwd(plan, qd, kd, vd)
    assert cp.check(plan) == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def _spiked_qkv(B, H, S, D, seed):
    """Scores with planted maxima that keep growing along the sequence: every
    query has a constant component along dimension 0 and every 97th key a large,
    increasing one there, so the running row max jumps by more than 2^8 (in the
    exp2 domain) many times, in the first and the second half of key tiles."""
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, S, H, D, generator=g)
    k = torch.randn(B, S, H, D, generator=g)
    v = torch.randn(B, S, H, D, generator=g)
    q[..., 0] = 4.0
    pos = torch.arange(5, S, 97)
    k[:, pos, :, 0] = (20.0 + 16.0 * torch.arange(len(pos), dtype=torch.float32))[None, :, None]
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


@pytest.mark.parametrize("layout,causal,D", [("zigzag", True, 128), ("contiguous", True, 128),
                                             ("contiguous", False, 128), ("zigzag", True, 64)])
def test_growing_row_max_rescales(layout, causal, D):
    q, k, v = _spiked_qkv(1, 2, 2048, D, 21)
    run_and_compare(q, k, v, 2, layout, causal, what=f"spiked {layout} causal={causal} D={D}")
