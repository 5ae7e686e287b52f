"""Failure detection and memory-safety checks on the GPU, none of which faults or hangs it.

* the bounded in-kernel wait runs out on a barrier nothing arrives on and the
  host reads CP_ERR_TIMEOUT; the context stays usable afterwards;
* outputs are written inside their bounds: guard regions around every output
  keep their sentinel bytes (a canary check in place of a sanitizer);
* misaligned or missing pointers are rejected before any launch.
"""
import numpy as np
import pytest
import torch

import context_long_sequence_cp_b200 as cp
from tests import gpu_util as G
from workloads import make_small

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    plan = cp.Plan(1, 2, 512, 128, 2, True, "zigzag")
    cp.debug_wait_timeout_probe(plan, 2000)          # 2 ms budget
    assert cp.check(plan) == -5
    assert cp.check(plan) == 0                       # the status word was cleared
    q, k, v = make_small(1, 2, 512, 128, 50)
    qd, kd, vd = (G.to_layout(x, 2, "zigzag").cuda() for x in (q, k, v))
    o, lse = cp.attn_fwd(plan, qd, kd, vd)
    assert cp.check(plan) == 0 and torch.isfinite(o.float()).all()


GUARD = 4096  # elements of guard before and after each output


def _guarded(shape, dtype, fill):
    n = int(np.prod(shape))
    buf = torch.full((GUARD + n + GUARD,), fill, dtype=dtype, device="cuda")
    return buf, buf[GUARD:GUARD + n].view(shape)


def _guards_intact(buf, n, fill):
    head, tail = buf[:GUARD], buf[GUARD + n:]
    return bool((head == fill).all()) and bool((tail == fill).all())


@pytest.mark.parametrize("B,H,S,D,N,layout,causal", [(1, 2, 800, 128, 4, "contiguous", True),
                                                     (2, 3, 384, 64, 3, "zigzag", True),
                                                     (2, 8, 512, 128, 4, "ulysses", False)])
def test_outputs_stay_in_bounds(B, H, S, D, N, layout, causal):
    q, k, v = make_small(B, H, S, D, 60)
    plan = cp.Plan(B, H, S, D, N, causal, layout)
    qd, kd, vd = (G.to_layout(x, N, layout).cuda() for x in (q, k, v))
    sent_o = torch.tensor(-12345.0, dtype=torch.bfloat16).item()
    obuf, o = _guarded(qd.shape, torch.bfloat16, sent_o)
    lbuf, lse = _guarded((B, H, S), torch.float32, 7777.0)
    cp.attn_fwd(plan, qd, kd, vd, o=o, lse=lse)
    assert cp.check(plan) == 0
    assert _guards_intact(obuf, o.numel(), sent_o)
    assert _guards_intact(lbuf, lse.numel(), 7777.0)
    assert not (o == sent_o).any() and not (lse == 7777.0).any()   # every element written
    if layout != "ulysses":
        rows = B * S * H
        pbuf, op = _guarded((N, rows, D), torch.float32, 555.0)
        lpbuf, lp = _guarded((N, rows), torch.float32, 555.0)
        cp.attn_fwd_partials(plan, qd, kd, vd, o_parts=op, lse_parts=lp)
        assert cp.check(plan) == 0
        assert _guards_intact(pbuf, op.numel(), 555.0) and _guards_intact(lpbuf, lp.numel(), 555.0)
        assert not (lp == 555.0).any()
        mbuf, om = _guarded((rows, D), torch.bfloat16, sent_o)
        cp.merge_partials(op, lp, o_out=om)
        torch.cuda.synchronize()
        assert _guards_intact(mbuf, om.numel(), sent_o)


def test_misaligned_and_null_pointers_rejected():
    plan = cp.Plan(1, 2, 512, 128, 2, True, "zigzag")
    x = torch.zeros(2 * 1 * 256 * 2 * 128 + 8, dtype=torch.bfloat16, device="cuda")
    good = x[:-8].view(2, 1, 256, 2, 128)
    bad = x[1:-7].view(2, 1, 256, 2, 128)            # 2-byte offset
    lib = cp.lib()
    P = lambda t: t.data_ptr()
    s = torch.cuda.current_stream().cuda_stream
    assert lib.cp_attn_fwd(plan.handle, P(bad), P(good), P(good), P(good), None, None, s) == -3
    assert lib.cp_attn_fwd(plan.handle, None, P(good), P(good), P(good), None, None, s) == -1
    assert lib.cp_layout_permute(plan.handle, 0, P(bad), P(good), 2, s) == -3
    assert lib.cp_layout_permute(plan.handle, 2, P(good), P(good), 2, s) == -1
    assert lib.cp_merge_partials(0, 10, 128, None, None, None, None, s) == -1
    assert lib.cp_merge_partials(2, 10, 96, P(good), P(good), P(good), None, s) == -2
    u = cp.Plan(1, 8, 512, 128, 4, False, "ulysses")
    assert lib.cp_attn_fwd(u.handle, P(good), P(good), P(good), P(good), None, None, s) == -6
