"""The Ulysses forward that allocates nothing, checked against cp_attn_fwd.

Callers that cannot call cudaMalloc at the point of the call (their device
memory belongs to another allocator, or allocation is not allowed there) use
cp_attn_fwd_ulysses_noalloc, which keeps its head-group copies in the
library's fixed device scratch instead of a caller workspace. This file is
collected last so that a run stopping at the first failure has run every
other test before it; it also passes on its own in a fresh process.
"""
import ctypes

import pytest
import torch

import context_long_sequence_cp_b200 as cp
from tests import gpu_util as G
from workloads import make_small

pytestmark = pytest.mark.gpu


def _noalloc(plan, q, k, v, o, lse):
    s = torch.cuda.current_stream().cuda_stream
    return cp.lib().cp_attn_fwd_ulysses_noalloc(plan.handle, ctypes.c_void_p(q.data_ptr()),
                                                ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
                                                ctypes.c_void_p(o.data_ptr()),
                                                None if lse is None else ctypes.c_void_p(lse.data_ptr()), s)


def _within(o, lse, o_ref, lse_ref):
    d = (o.float() - o_ref.float()).abs()
    assert d.max().item() <= G.TOL_O_MAX and d.mean().item() <= G.TOL_O_MEAN
    assert (lse - lse_ref).abs().max().item() <= G.TOL_LSE


def test_noalloc_matches_workspace_path_on_two_calls_in_a_row():
    B, H, S, D, N = 2, 8, 1024, 128, 4                 # needs 16 MiB of scratch
    plan = cp.Plan(B, H, S, D, N, False, "ulysses")
    assert plan.workspace_bytes() <= cp.NOALLOC_SCRATCH_BYTES
    inputs, refs = [], []
    for seed in (71, 72):
        q, k, v = make_small(B, H, S, D, seed)
        qd, kd, vd = (G.to_layout(x, N, "ulysses").cuda() for x in (q, k, v))
        inputs.append((qd, kd, vd))
        refs.append(cp.attn_fwd(plan, qd, kd, vd))      # the existing entry point, with a workspace
    assert cp.check(plan) == 0
    outs = []
    for qd, kd, vd in inputs:                          # two no-alloc calls back to back
        o = torch.empty_like(qd)
        lse = torch.empty(B, H, S, dtype=torch.float32, device="cuda")
        assert _noalloc(plan, qd, kd, vd, o, lse) == 0
        outs.append((o, lse))
    assert cp.check(plan) == 0
    for (o, lse), (o_ref, lse_ref) in zip(outs, refs):
        _within(o, lse, o_ref, lse_ref)


def test_noalloc_rejects_oversize_and_other_layouts():
    big = cp.Plan(2, 32, 16384, 128, 8, False, "ulysses")   # needs 1 GiB > 32 MiB
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(big, x, x, x, x, None) == -6            # CP_ERR_WORKSPACE, nothing launched
    zz = cp.Plan(1, 2, 512, 128, 2, True, "zigzag")
    assert _noalloc(zz, x, x, x, x, None) == -2             # CP_ERR_UNSUPPORTED
    assert cp.check(zz) == 0
