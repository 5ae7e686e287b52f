"""GPU parity of the RoPE-fused layout map (cp_rope_permute) against the fp64 oracle,
and of attention on rotated Q/K against the oracle's attention of rope(Q), rope(K).

Tolerance per element, from the arithmetic: the kernel rotates bf16 inputs in fp32
with sincosf of an fp64-reduced angle (error ~1e-6 of the pair's norm) and rounds
once to bf16 (at most one ulp, 2^-8 relative, when the fp32 error crosses a
rounding boundary): |gpu - oracle| <= 2^-8 |oracle| + 1e-5 * |pair|.
"""
import numpy as np
import pytest
import torch

import context_long_sequence_cp_b200 as cp
from oracle import layouts as L
from oracle import rope as R
from tests import gpu_util as G
from workloads import WORKLOADS, make_qkv, make_small, sample_rows

pytestmark = pytest.mark.gpu


def natural_rope(x, offset, base=10000.0):
    """Oracle: rope of natural [B, S, H, D] at global positions s + offset (fp64)."""
    B, S, H, D = x.shape
    xn = x.float().numpy()
    return np.stack([R.rope(xn[b], np.arange(S) + offset, base) for b in range(B)])


def assert_rope_close(gpu, ref):
    """gpu, ref: [..., D] fp64 arrays."""
    pair = np.sqrt(ref[..., 0::2] ** 2 + ref[..., 1::2] ** 2)
    bound = np.empty_like(ref)
    bound[..., 0::2] = 2.0 ** -8 * np.abs(ref[..., 0::2]) + 1e-5 * pair
    bound[..., 1::2] = 2.0 ** -8 * np.abs(ref[..., 1::2]) + 1e-5 * pair
    err = np.abs(gpu - ref)
    assert np.all(err <= bound), float((err - bound).max())


def view_to_natural(y, B, S, H, N, layout):
    """Attention-input layout -> natural [B, S, H, D] fp64 (oracle index maps)."""
    D = y.shape[-1]
    if layout == "ulysses":
        # groups [N, B, S, H/N, D]: group g holds heads g*H/N ..
        g = y.reshape(N, B, S, H // N, D).permute(1, 2, 0, 3, 4).reshape(B, S, H, D)
        return g.double().cpu().numpy()
    m = L.rank_major_map(B, S, N, layout)           # rank-major row -> natural row
    nat = torch.empty(B * S, H, D, dtype=y.dtype, device=y.device)
    nat[torch.from_numpy(m).to(y.device)] = y.reshape(B * S, H, D)
    return nat.reshape(B, S, H, D).double().cpu().numpy()


@pytest.mark.parametrize("B,H,S,D,N,layout,offset", [
    (1, 2, 256, 64, 4, "contiguous", 0),
    (2, 3, 1024, 128, 2, "zigzag", 0),
    (1, 4, 512, 128, 4, "zigzag", 123457),
    (2, 8, 512, 64, 4, "ulysses", 0),
    (1, 2, 256, 128, 2, "contiguous", (1 << 31) - 256),   # largest allowed positions
])
def test_rope_permute_all_elements(B, H, S, D, N, layout, offset):
    q, _, _ = make_small(B, H, S, D, seed=31)
    plan = cp.Plan(B, H, S, D, N, True if layout != "ulysses" else False, layout)
    x = (G.to_layout(q, N, "contiguous") if layout == "ulysses" else q).cuda()
    y = cp.rope_permute(plan, x, pos_offset=offset)
    assert cp.check(plan) == 0
    gpu = view_to_natural(y, B, S, H, N, layout)
    assert_rope_close(gpu, natural_rope(q, offset))
    plan.close()


def test_rope_permute_zigzag_32k_sampled_rows():
    w = WORKLOADS["zigzag_32k"]
    q, _, _ = make_qkv(w)
    plan = cp.Plan(w.B, w.H, w.S, w.D, w.N, w.causal, w.layout)
    y = cp.rope_permute(plan, q.cuda())
    assert cp.check(plan) == 0
    rows = sample_rows(w)
    got = G.gather_rows(y, w.B, w.S, w.H, w.N, w.layout, rows)            # [n, D]
    xs = q.float().numpy()[rows[:, 0], rows[:, 2], rows[:, 1]]             # [n, D]
    ref = np.stack([R.rope(xs[i][None, None], np.array([rows[i, 2]]))[0, 0] for i in range(len(rows))])
    assert_rope_close(got, ref)
    plan.close()


def test_rope_then_attention_matches_oracle():
    # The pages' point: positions must be global. Attention on rope'd Q/K from the
    # zigzag layout equals the oracle's attention of rope(Q), rope(K) in natural order.
    B, H, S, D, N = 1, 2, 1024, 128, 4
    q, k, v = make_small(B, H, S, D, seed=32)
    plan = cp.Plan(B, H, S, D, N, True, "zigzag")
    qz = cp.rope_permute(plan, q.cuda())
    kz = cp.rope_permute(plan, k.cuda())
    vz = cp.layout_permute(plan, v.cuda(), 0)
    o, lse = cp.attn_fwd(plan, qz, kz, vz)
    assert cp.check(plan) == 0
    # Oracle inputs: the bf16-rounded rotated values the attention actually saw
    # would hide a position bug, so rotate in fp64 and compare within the
    # attention tolerance (the bf16 rounding of Q/K is far inside it).
    qr = torch.from_numpy(natural_rope(q, 0)).to(torch.bfloat16)
    kr = torch.from_numpy(natural_rope(k, 0)).to(torch.bfloat16)
    bb, hh, ii = np.meshgrid(np.arange(B), np.arange(H), np.arange(S), indexing="ij")
    rows = np.stack([bb.ravel(), hh.ravel(), ii.ravel()], 1).astype(np.int64)
    o_gpu = G.gather_rows(o, B, S, H, N, "zigzag", rows)
    lse_gpu = lse.cpu().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]].astype(np.float64)
    o_ref, lse_ref = G.oracle_rows(qr, kr, v, rows, True)
    G.assert_within(G.errors(o_gpu, o_ref, lse_gpu, lse_ref), "rope + attention")
    plan.close()
