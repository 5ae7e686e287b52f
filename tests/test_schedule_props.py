"""Property tests of the C library's host-side schedules (no GPU): over random
plan shapes, every schedule covers its work exactly once and its modelled loads
add up.

Page "序列与上下文并行", section "上下文并行：注意力本身切分": rank r at ring step
t works on the key/value block of rank (r + t) mod N; a causal query only sees
keys at or before its global position. Brute force over the layout's positions
(oracle.layouts) decides which (query tile, key tile) pairs a walk must visit.
"""
import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import context_long_sequence_cp_b200 as cp
from context_long_sequence_cp_b200 import build as cpbuild
from oracle.layouts import chunk_positions

TILE = 128


@pytest.fixture(scope="module", autouse=True)
def built():
    cpbuild.build()


@st.composite
def plans(draw):
    N = draw(st.integers(1, 6))
    layout = draw(st.sampled_from(["contiguous", "zigzag"]))
    unit = 2 * N if layout == "zigzag" else N
    # local lengths from a few tokens to several tiles, ragged included
    S = unit * draw(st.integers(1, 1200 // unit + 1))
    B = draw(st.integers(1, 2))
    H = draw(st.integers(1, 3))
    D = draw(st.sampled_from([64, 128]))
    causal = draw(st.booleans())
    return B, H, S, D, N, causal, layout


def _walks(S, N, layout, causal):
    """walk[r][t][qp]: key tiles of block (r + t) mod N that query-tile pair qp of
    rank r visits (a key tile counts when either query tile has an allowed key)."""
    pos = chunk_positions(S, N, layout)
    T = S // N
    nt = -(-T // TILE)
    tiles = lambda r: [pos[r, i * TILE:(i + 1) * TILE] for i in range(nt)]
    out = []
    for r in range(N):
        qt = tiles(r)
        per_t = []
        for t in range(N):
            kt = tiles((r + t) % N)
            row = []
            for qp in range(-(-nt // 2)):
                n = 0
                for kk in kt:
                    n += any((not causal) or kk.min() <= qq.max() for qq in qt[2 * qp:2 * qp + 2])
                row.append(n)
            per_t.append(row)
        out.append(per_t)
    return out


@settings(max_examples=25, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(plans())
def test_every_schedule_covers_its_work_once(shape):
    B, H, S, D, N, causal, layout = shape
    p = cp.Plan(B, H, S, D, N, causal, layout)
    T = S // N
    npairs = -(-T // (2 * TILE))
    walks = _walks(S, N, layout, causal)

    # the fused kernel's static schedule: every walked key tile and item once
    walked = sum(walks[r][t][qp] for r in range(N) for t in range(N) for qp in range(npairs)) * B * H
    loads = np.array(p.cta_loads())
    assert p.num_items() == N * B * H * npairs
    assert loads.sum() == 2 * walked + 3 * p.num_items()
    assert loads.max() <= loads.mean() + 2 * max(sum(walks[r][t][qp] for t in range(N))
                                                  for r in range(N) for qp in range(npairs)) + 3

    split = N if N <= 2 else (N + 1) // 2
    assert p.ring_parts() == (split + 1 if split < N else N)
    for r in range(N):
        # per-step schedules: each (b, h, pair) once, its walk at that step
        for t in range(N):
            items, sl = p.ring_schedule(r, t)
            assert sorted((rb, h, qp) for rb, h, qp, _, _ in items) == sorted(
                (r * B + b, h, qp) for b in range(B) for h in range(H) for qp in range(npairs))
            assert all(cost == walks[r][t][qp] for _, _, qp, cost, _ in items)
            assert sum(sl) == sum(2 * it[3] + 3 for it in items)
        # one-launch units: every step of every pair once, phases in order per CTA
        units, ul = p.ring_schedule(r, -1)
        cover = {}
        for rb, h, q, cost, cta in units:
            qp, t0, t1 = q & 0xffff, (q >> 16) & 0xff, (q >> 24) & 0xff
            assert cost == sum(walks[r][t][qp] for t in range(t0, t1))
            cover.setdefault((rb, h, qp), []).extend(range(t0, t1))
        assert set(cover) == {(r * B + b, h, qp) for b in range(B) for h in range(H) for qp in range(npairs)}
        assert all(sorted(v) == list(range(N)) for v in cover.values())
        for c in set(u[4] for u in units):
            phases = [(u[2] >> 16) & 0xff for u in units if u[4] == c]
            assert phases == sorted(phases)
        assert sum(ul) == sum(2 * u[3] + 3 for u in units)
