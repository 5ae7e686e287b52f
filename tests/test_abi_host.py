"""Host-side checks of the C ABI: no GPU needed, no compute calls.

* the library builds, loads and exports every function ``include/cp_attn.h`` declares;
* plan creation validates its arguments;
* the plan's executed tile-pair counts equal the oracle's brute-force enumeration.
"""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import context_long_sequence_cp_b200 as cp
from context_long_sequence_cp_b200 import build as cpbuild
from oracle import schedule as Sch
from workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "cp_attn.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    cpbuild.build()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(cp_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("cp_attn_plan", "cp_attn_fwd", "cp_merge_partials", "cp_layout_permute",
                     "cp_layout_index_map", "cp_attn_fwd_partials", "cp_attn_check"):
        assert required in names
    assert sorted(cp.SIGNATURES) == names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", cp.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(\S+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        assert getattr(cp.lib(), name) is not None
    # nothing else leaks out of the library's C++/CUDA internals
    assert not [s for s in exported if s.startswith("_ZN6cpattn")]


def test_status_strings():
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert cp.status_string(code) not in ("", "unknown status")
    assert cp.status_string(-99) == "unknown status"


def _plan_status(*args):
    h = ctypes.c_void_p()
    rc = cp.lib().cp_attn_plan(ctypes.byref(h), *args)
    if rc == 0:
        cp.lib().cp_attn_plan_destroy(h)
    else:
        assert h.value is None
    return rc


def test_plan_argument_validation():
    Z, C, U = cp.ZIGZAG, cp.CONTIGUOUS, cp.ULYSSES
    assert _plan_status(1, 2, 256, 64, 4, 0, C, 0.0) == 0
    assert _plan_status(1, 2, 256, 96, 4, 0, C, 0.0) == -2          # D not 64/128
    assert _plan_status(1, 2, 250, 64, 4, 0, C, 0.0) == -2          # S % N
    assert _plan_status(1, 2, 255, 64, 5, 1, Z, 0.0) == -2          # S % 2N for zigzag
    assert _plan_status(1, 6, 256, 64, 4, 0, U, 0.0) == -2          # H % N for Ulysses
    assert _plan_status(1, 8, 256, 64, 4, 1, U, 0.0) == -2          # causal Ulysses
    assert _plan_status(0, 2, 256, 64, 4, 0, C, 0.0) == -1          # B <= 0
    assert _plan_status(1, 2, 256, 64, 0, 0, C, 0.0) == -1          # N <= 0
    assert _plan_status(1, 2, 256, 64, 4, 2, C, 0.0) == -1          # causal not 0/1
    assert _plan_status(1, 2, 256, 64, 4, 0, 7, 0.0) == -1          # bad layout
    assert cp.lib().cp_attn_plan(None, 1, 2, 256, 64, 4, 0, C, 0.0) == -1
    assert cp.lib().cp_attn_plan_destroy(None) == 0


def test_plan_size_limits():
    """Shapes beyond what the kernels index are refused up front, before any table
    is built: the packed walk entries (key rank < 2^12, key tile < 2^13), the
    view's row blocks (B * N <= 2^20) and the element count (<= 2^40)."""
    C = cp.CONTIGUOUS
    assert _plan_status(1, 0, 256, 64, 4, 0, C, 0.0) == -1                # H <= 0
    assert _plan_status(1, 2, 0, 64, 4, 0, C, 0.0) == -1                  # S <= 0
    assert _plan_status(1, 2, 256, 64, 4, 0, C, float("nan")) == -1       # scale NaN
    assert _plan_status(1, 2, 256, 64, 4, 0, C, float("inf")) == -1       # scale inf
    assert _plan_status(1, 1, 4096, 64, 4096, 0, C, 0.0) == -2            # N = 2^12 ranks
    assert _plan_status(1, 1, 8192 * 128, 64, 1, 0, C, 0.0) == -2         # 2^13 key tiles
    assert _plan_status(1 << 18, 1, 8, 64, 8, 0, C, 0.0) == -2            # B * N = 2^21
    assert _plan_status(1024, 1024, 1 << 16, 128, 1, 0, C, 0.0) == -2     # 2^43 elements
    assert _plan_status(1, 2, 256, 64, 4, 0, C, 0.5) == 0                 # explicit scale


@pytest.mark.parametrize("S,N,layout,causal", [
    (32768, 8, "zigzag", True), (32768, 8, "contiguous", True), (4096, 4, "zigzag", True),
    (131072, 4, "zigzag", True), (131072, 4, "contiguous", True), (256, 4, "contiguous", False),
    (800, 4, "contiguous", True), (384, 3, "zigzag", True), (1000, 5, "zigzag", True),
])
def test_plan_tile_counts_match_oracle(S, N, layout, causal):
    B, H = 2, 3
    plan = cp.Plan(B, H, S, 128, N, causal, layout)
    per_rank, total = plan.tile_counts()
    ref = Sch.tile_pair_counts(S, N, layout, causal) * B * H
    assert per_rank == [int(x) for x in ref]
    assert total == int(ref.sum())
    plan.close()


def test_plan_zigzag_balance_and_contiguous_imbalance():
    w = WORKLOADS["zigzag_32k"]
    z = cp.Plan(w.B, w.H, w.S, w.D, w.N, True, "zigzag").tile_counts()[0]
    c = cp.Plan(w.B, w.H, w.S, w.D, w.N, True, "contiguous").tile_counts()[0]
    assert len(set(z)) == 1 and z[0] == 4112 * w.H
    assert abs(max(c) / (sum(c) / len(c)) - 1.8716) < 1e-4


def test_workspace_and_map_sizes():
    p = cp.Plan(2, 32, 16384, 128, 8, False, "ulysses")
    assert p.workspace_bytes(False) == 4 * 2 * 16384 * 32 * 128 * 2
    assert p.index_map_len() == 8 * 2 * 16384
    assert p.tile_counts()[0] == [2 * 4 * 128 * 128] * 8
    z = cp.Plan(1, 16, 4096, 128, 4, True, "zigzag")
    assert z.workspace_bytes(False) == 0 and z.workspace_bytes(True) == 0
    assert z.index_map_len() == 4096
    assert z.num_items() == 4 * 16 * 4     # ranks x heads x query-tile pairs (T=1024)


def _executed_key_tiles(S, N, layout, causal, tile=128):
    """Key tiles walked per (batch, head): a key tile counts once per query-tile
    pair in which at least one of the two query tiles has an allowed key in it."""
    from oracle.layouts import chunk_positions
    pos = chunk_positions(S, N, layout)
    T = S // N
    nt = -(-T // tile)
    tmin = np.array([[pos[r, i * tile:(i + 1) * tile].min() for i in range(nt)] for r in range(N)])
    tmax = np.array([[pos[r, i * tile:(i + 1) * tile].max() for i in range(nt)] for r in range(N)])
    total = 0
    for r in range(N):
        for t in range(N):
            rk = (r + t) % N
            ok = tmin[rk][None, :] <= tmax[r][:, None] if causal else np.ones((nt, nt), bool)
            for qp in range(-(-nt // 2)):
                rows = ok[2 * qp:2 * qp + 2]
                total += int(rows.any(axis=0).sum())
    return total


@pytest.mark.parametrize("layout", ["zigzag", "contiguous"])
def test_static_schedule_is_balanced_and_complete(layout):
    w = WORKLOADS["zigzag_32k"]
    p = cp.Plan(w.B, w.H, w.S, w.D, w.N, True, layout)
    loads = np.array(p.cta_loads())
    assert len(loads) == 148                        # one CTA per SM (no device here: 148)
    assert loads.max() / loads.mean() < 1.02
    # Modelled load = 2 per walked key tile + 3 per item, so the loads add up to
    # the work of every item exactly once.
    walked = _executed_key_tiles(w.S, w.N, layout, True) * w.H
    assert loads.sum() == 2 * walked + 3 * p.num_items()


def test_static_schedule_few_items_per_cta_is_longest_first():
    # zigzag_4k: 256 items on 148 CTAs. Grouping items by head pair would leave the
    # late groups' long items on CTAs already holding short ones (modelled max/mean
    # 1.59); the longest-first assignment ends at the largest single item.
    w = WORKLOADS["zigzag_4k"]
    p = cp.Plan(w.B, w.H, w.S, w.D, w.N, True, "zigzag")
    loads = np.array(p.cta_loads())
    walked = _executed_key_tiles(w.S, w.N, "zigzag", True) * w.H
    assert loads.sum() == 2 * walked + 3 * p.num_items()
    largest_item = 2 * (w.S // 128) + 3          # the last pair walks every key tile
    assert loads.max() == largest_item
    assert loads.max() / loads.mean() < 1.05


def test_static_schedule_small_plan_one_item_per_cta():
    p = cp.Plan(1, 2, 256, 64, 4, False, "contiguous")   # 4 ranks x 2 heads x 1 pair
    loads = p.cta_loads()
    assert len(loads) == p.num_items() == 8
    # Non-causal: every item walks all 4 ranks' single key tile.
    assert loads == [2 * 4 + 3] * 8


def test_rope_permute_argument_validation():
    # Host-side checks run before any device work (no GPU here: valid calls end
    # in CP_ERR_CUDA).
    L = cp.lib()
    p = cp.Plan(1, 2, 256, 64, 4, True, "zigzag")
    ok_in, ok_out = ctypes.c_void_p(4096), ctypes.c_void_p(8192)
    assert L.cp_rope_permute(None, ok_in, ok_out, 10000.0, 0, None) == -1
    assert L.cp_rope_permute(p.handle, None, ok_out, 10000.0, 0, None) == -1
    assert L.cp_rope_permute(p.handle, ok_in, None, 10000.0, 0, None) == -1
    assert L.cp_rope_permute(p.handle, ok_in, ok_out, 1.0, 0, None) == -1        # base must be > 1
    assert L.cp_rope_permute(p.handle, ok_in, ok_out, float("nan"), 0, None) == -1
    assert L.cp_rope_permute(p.handle, ok_in, ok_out, 10000.0, -1, None) == -1   # negative offset
    assert L.cp_rope_permute(p.handle, ok_in, ok_out, 10000.0, (1 << 31) - 255, None) == -1
    assert L.cp_rope_permute(p.handle, ctypes.c_void_p(4100), ok_out, 10000.0, 0, None) == -3   # alignment
    assert L.cp_rope_permute(p.handle, ok_in, ok_out, 10000.0, (1 << 31) - 256, None) in (0, -4)
    p.close()


@pytest.mark.parametrize("S,N,layout,causal", [
    (32768, 8, "zigzag", True), (4096, 4, "zigzag", True), (800, 4, "contiguous", True),
    (256, 4, "contiguous", False), (384, 3, "zigzag", True),
])
def test_bwd_walks_cover_every_executed_tile_pair(S, N, layout, causal):
    # Both backward walks visit exactly the executed (query tile, key tile)
    # pairs of the forward, counted by brute force in the oracle.
    p = cp.Plan(1, 2, S, 128, N, causal, layout)
    kv, qq = p.bwd_pairs()
    ref = int(Sch.tile_pair_counts(S, N, layout, causal).sum())
    assert kv == qq == ref
    rows = N * 1 * (S // N) * 2
    assert p.bwd_workspace_bytes() == 2 * rows * 4 + 1024
    p.close()


def test_bwd_argument_validation():
    L = cp.lib()
    p = cp.Plan(1, 2, 256, 64, 4, True, "zigzag")
    a = [ctypes.c_void_p(4096 * (i + 1)) for i in range(10)]
    assert L.cp_attn_bwd(None, *a, None) == -1
    for i in range(10):
        b = list(a)
        b[i] = None
        assert L.cp_attn_bwd(p.handle, *b, None) == -1, i
    b = list(a)
    b[3] = ctypes.c_void_p(4100)
    assert L.cp_attn_bwd(p.handle, *b, None) == -3                  # alignment
    assert L.cp_attn_bwd(p.handle, *a, None) in (0, -4)             # no device here
    u = cp.Plan(2, 8, 256, 64, 4, False, "ulysses")
    assert L.cp_attn_bwd(u.handle, *a, None) == -2                  # no Ulysses backward
    assert u.bwd_workspace_bytes() == 0
    p.close()
    u.close()


def test_sp_rs_dropout_add_ln_argument_validation():
    L = cp.lib()
    P = lambda a: ctypes.c_void_p(a)
    pt, z, y, g, b, kb = P(4096), P(8192), P(12288), P(16384), P(20480), P(24576)
    f = L.cp_sp_rs_dropout_add_ln
    assert f(None, 1, 4, 64, None, 0.0, None, None, None, 1e-5, z, None, None) == -1
    assert f(pt, 0, 4, 64, None, 0.0, None, None, None, 1e-5, z, None, None) == -1      # nparts < 1
    assert f(pt, 1, 4, 60, None, 0.0, None, None, None, 1e-5, z, None, None) == -2      # H % 8
    assert f(pt, 1, 4, 16384, None, 0.0, None, None, None, 1e-5, z, None, None) == -2   # H > 8192
    assert f(pt, 1, 4, 64, kb, 1.0, None, None, None, 1e-5, z, None, None) == -1        # p must be < 1
    assert f(pt, 1, 4, 64, None, 0.0, None, g, None, 1e-5, z, None, None) == -1        # gamma without beta
    assert f(pt, 1, 4, 64, None, 0.0, None, None, None, 1e-5, None, y, None) == -1     # y needs gamma
    assert f(pt, 1, 4, 64, None, 0.0, None, None, None, 1e-5, None, None, None) == -1  # no output
    assert f(pt, 1, 4, 64, None, 0.0, None, g, b, 0.0, None, y, None) == -1           # eps > 0
    assert f(P(4100), 1, 4, 64, None, 0.0, None, None, None, 1e-5, z, None, None) == -3
    assert f(pt, 1, 4, 64, P(24578), 0.1, None, None, None, 1e-5, z, None, None) == -3  # keep bits 4-aligned
    assert f(pt, 2, 4, 64, kb, 0.1, None, g, b, 1e-5, z, y, None) in (0, -4)           # no device here
