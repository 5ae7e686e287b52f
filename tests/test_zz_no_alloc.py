"""The Ulysses forward that allocates nothing, checked against cp_attn_fwd.

Callers that cannot call cudaMalloc at the point of the call (their device
memory belongs to another allocator, or allocation is not allowed there) use
cp_attn_fwd_ulysses_noalloc, which keeps its head-group copies in the
library's fixed device scratch instead of a caller workspace. It runs the same
kernels on the same inputs as cp_attn_fwd, so its results must be bit-identical
to that entry point's; one call's rows are also compared with the fp64 oracle.
This file is collected last so that a run stopping at the first failure has run
every other test before it; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
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


def test_noalloc_matches_workspace_path_on_two_calls_in_a_row():
    B, H, S, D, N = 2, 8, 1024, 128, 4                 # needs 16 MiB of scratch
    plan = cp.Plan(B, H, S, D, N, False, "ulysses")
    assert plan.workspace_bytes() <= cp.NOALLOC_SCRATCH_BYTES
    inputs, refs, nat = [], [], []
    for seed in (71, 72):
        q, k, v = make_small(B, H, S, D, seed)
        nat.append((q, k, v))
        qd, kd, vd = (G.to_layout(x, N, "ulysses").cuda() for x in (q, k, v))
        inputs.append((qd, kd, vd))
        refs.append(cp.attn_fwd(plan, qd, kd, vd))      # the existing entry point, with a workspace
    assert cp.check(plan) == 0
    outs = []
    for i, (qd, kd, vd) in enumerate(inputs):          # two no-alloc calls back to back
        o = torch.full_like(qd, float("nan"))
        lse = torch.full((B, H, S), float("nan"), dtype=torch.float32, device="cuda")
        if i == 0:
            assert _noalloc(plan, qd, kd, vd, o, lse) == 0          # raw through the C ABI
        else:
            cp.attn_fwd_ulysses_noalloc(plan, qd, kd, vd, o, lse)   # through the binding
        outs.append((o, lse))
    assert cp.check(plan) == 0
    for (o, lse), (o_ref, lse_ref) in zip(outs, refs):
        # same kernels, same inputs: bit-identical (a scratch-aliasing bug would not be)
        assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16))
        assert torch.equal(lse.view(torch.int32), lse_ref.view(torch.int32))
    # the second call's rows against the fp64 oracle, within the attention tolerances
    q, k, v = nat[1]
    rng = np.random.default_rng(7)
    rows = np.stack([rng.integers(0, B, 256), rng.integers(0, H, 256), rng.integers(0, S, 256)], 1)
    o_gpu = G.gather_rows(outs[1][0], B, S, H, N, "ulysses", rows)
    lse_gpu = outs[1][1].cpu().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]].astype(np.float64)
    o_ref, lse_ref = G.oracle_rows(q, k, v, rows, causal=False)
    G.assert_within(G.errors(o_gpu, o_ref, lse_gpu, lse_ref), "no-alloc vs oracle")


def test_noalloc_rejects_oversize_other_layouts_and_bad_arguments():
    big = cp.Plan(2, 32, 16384, 128, 8, False, "ulysses")   # needs 1 GiB > 32 MiB
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(big, x, x, x, x, None) == -6            # CP_ERR_WORKSPACE, nothing launched
    zz = cp.Plan(1, 2, 512, 128, 2, True, "zigzag")
    assert _noalloc(zz, x, x, x, x, None) == -2             # CP_ERR_UNSUPPORTED
    assert cp.check(zz) == 0
    small = cp.Plan(1, 4, 256, 64, 2, False, "ulysses")
    good = torch.zeros(2, 1, 128, 4, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):                         # wrong shape, caught by the binding
        cp.attn_fwd_ulysses_noalloc(small, x, good, good, good)
    with pytest.raises(ValueError):                         # wrong dtype
        cp.attn_fwd_ulysses_noalloc(small, good.float(), good, good, good)
    with pytest.raises(ValueError):                         # undersized lse
        cp.attn_fwd_ulysses_noalloc(small, good, good, good, torch.empty_like(good),
                                    torch.empty(4, dtype=torch.float32, device="cuda"))
