"""Layout maps of the oracle pinned against hand-derived golden examples and bijectivity."""
import os

import numpy as np
import pytest

from oracle import layouts as L
from oracle import schedule as Sch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        rows = [ln for ln in f if ln.strip() and not ln.startswith("#")]
    return np.array(rows[0].split(), dtype=np.int64)


def test_zigzag_worked_example():
    np.testing.assert_array_equal(L.rank_major_map(1, 16, 2, "zigzag"), _golden("zigzag_S16_N2.txt"))


def test_contiguous_worked_example():
    np.testing.assert_array_equal(L.rank_major_map(2, 8, 4, "contiguous"),
                                  _golden("contiguous_S8_N4_B2.txt"))


def test_ulysses_worked_example():
    np.testing.assert_array_equal(L.ulysses_run_map(1, 4, 4, 2), _golden("ulysses_N2_B1_S4_H4.txt"))


@pytest.mark.parametrize("B,S,N,layout", [(1, 16, 2, "zigzag"), (2, 48, 3, "zigzag"),
                                          (3, 20, 5, "contiguous"), (1, 4096, 4, "zigzag"),
                                          (1, 32768, 8, "zigzag")])
def test_rank_major_map_is_bijection(B, S, N, layout):
    m = L.rank_major_map(B, S, N, layout)
    assert np.array_equal(np.sort(m), np.arange(B * S))


def test_rank_major_roundtrip_and_positions():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((2, 24, 3, 2))
    for layout in ("contiguous", "zigzag"):
        y = L.to_rank_major(x, 3, layout)
        np.testing.assert_array_equal(L.from_rank_major(y, layout), x)
    # zigzag: local token j < C of rank r is global r*C + j, j >= C is (2N-1-r)*C + j - C
    pos = L.chunk_positions(24, 3, "zigzag")
    C = 4
    for r in range(3):
        for j in range(8):
            exp = r * C + j if j < C else (5 - r) * C + j - C
            assert pos[r, j] == exp
    # positions within a rank increase monotonically (both layouts)
    for layout in ("contiguous", "zigzag"):
        assert np.all(np.diff(L.chunk_positions(64, 4, layout), axis=1) > 0)


@pytest.mark.parametrize("B,S,H,N", [(1, 4, 4, 2), (2, 16, 8, 4), (2, 64, 32, 8)])
def test_ulysses_bijection_and_roundtrip(B, S, H, N):
    m = L.ulysses_run_map(B, S, H, N)
    assert np.array_equal(np.sort(m), np.arange(N * B * S))
    rng = np.random.default_rng(1)
    x = rng.standard_normal((N, B, S // N, H, 3))
    g = L.shards_to_groups(x, N)
    # group g, batch b, token s holds heads g*H/N.. of the shard that owns s
    Hg = H // N
    for gi in range(N):
        for b in range(B):
            for s in range(S):
                rho, sl = divmod(s, S // N)
                np.testing.assert_array_equal(g[gi, b, s], x[rho, b, sl, gi * Hg:(gi + 1) * Hg])
    np.testing.assert_array_equal(L.groups_to_shards(g), x)


def test_schedule_closed_forms():
    """Executed 128x128 tile pairs per rank (per batch, head) against closed forms.

    With c = C/128 tiles per chunk, a same-chunk (diagonal) pair executes
    c(c+1)/2 tiles and an earlier-chunk pair c^2; summed over ranks the causal
    total is n(n+1)/2 for n = S/128 tiles.
    """
    z = Sch.tile_pair_counts(32768, 8, "zigzag", True)
    assert list(z) == [4112] * 8 and z.sum() == 256 * 257 // 2
    c = Sch.tile_pair_counts(32768, 8, "contiguous", True)
    assert list(c) == [1024 * r + 528 for r in range(8)]
    assert abs(Sch.imbalance(c) - 1.8716) < 1e-4 and Sch.imbalance(z) == 1.0
    z4 = Sch.tile_pair_counts(131072, 4, "zigzag", True)
    assert list(z4) == [131200] * 4 and z4.sum() == 1024 * 1025 // 2
    c4 = Sch.tile_pair_counts(131072, 4, "contiguous", True)
    assert list(c4) == [32896, 98432, 163968, 229504]
    assert abs(Sch.imbalance(c4) - 1.7493) < 1e-4
    assert list(Sch.tile_pair_counts(4096, 4, "zigzag", True)) == [132] * 4
    # non-causal: every rank executes (T/128)^2 * N pairs
    assert list(Sch.tile_pair_counts(256, 4, "contiguous", False)) == [4] * 4
