"""GPU checks of the HBM-bound kernels against the oracle.

* layout permutation and index map: bit-exact against the oracle's NumPy fancy
  indexing (compared as int16 / int32 bit patterns), round trips are identities;
* merge of partials: against the oracle's fp64 merge, with empty (-inf) partials;
* unfused partials + merge: each step's partial against the oracle's ring
  partial, and the merged result against the fused kernel.
"""
import numpy as np
import pytest
import torch

import context_long_sequence_cp_b200 as cp
from oracle import attention as A
from oracle import layouts as L
from tests import gpu_util as G
from workloads import WORKLOADS, make_qkv, make_small

pytestmark = pytest.mark.gpu

LAYOUT_CASES = [
    (1, 16, 4096, 128, 4, "zigzag"),
    (2, 4, 1536, 64, 3, "zigzag"),
    (3, 2, 800, 128, 4, "contiguous"),
    (1, 32, 32768, 128, 8, "zigzag"),
]


@pytest.mark.parametrize("B,H,S,D,N,layout", LAYOUT_CASES)
def test_rank_major_permute_bit_exact(B, H, S, D, N, layout):
    plan = cp.Plan(B, H, S, D, N, layout == "zigzag", layout)
    m = cp.layout_index_map(plan).cpu().numpy()
    np.testing.assert_array_equal(m, L.rank_major_map(B, S, N, layout))
    g = torch.Generator().manual_seed(5)
    x = torch.randn(B, S, H, D, generator=g).to(torch.bfloat16)
    y = cp.layout_permute(plan, x.cuda(), 0)
    ref = L.to_rank_major(x.view(torch.int16).numpy(), N, layout)
    np.testing.assert_array_equal(y.view(torch.int16).cpu().numpy().reshape(ref.shape), ref)
    back = cp.layout_permute(plan, y, 1)
    assert torch.equal(back.view(torch.int16).cpu(), x.view(torch.int16))
    # 4-byte elements
    xf = torch.randn(B, S, H, D, generator=g)
    yf = cp.layout_permute(plan, xf.cuda(), 0)
    reff = L.to_rank_major(xf.view(torch.int32).numpy(), N, layout)
    np.testing.assert_array_equal(yf.view(torch.int32).cpu().numpy().reshape(reff.shape), reff)


@pytest.mark.parametrize("B,S,H,D,N", [(1, 4, 4, 64, 2), (2, 512, 8, 128, 4), (2, 16384, 32, 128, 8)])
def test_ulysses_permute_bit_exact(B, S, H, D, N):
    plan = cp.Plan(B, H, S, D, N, False, "ulysses")
    m = cp.layout_index_map(plan).cpu().numpy()
    np.testing.assert_array_equal(m, L.ulysses_run_map(B, S, H, N))
    g = torch.Generator().manual_seed(6)
    x = torch.randn(N, B, S // N, H, D, generator=g).to(torch.bfloat16)
    y = cp.layout_permute(plan, x.cuda(), 0)
    ref = L.shards_to_groups(x.view(torch.int16).numpy(), N)
    np.testing.assert_array_equal(y.view(torch.int16).cpu().numpy().reshape(ref.shape), ref)
    back = cp.layout_permute(plan, y, 1)
    assert torch.equal(back.view(torch.int16).cpu(), x.view(torch.int16))


@pytest.mark.parametrize("P,rows,D", [(1, 1000, 128), (4, 4097, 64), (8, 20000, 128), (3, 5, 64)])
def test_merge_kernel_vs_oracle(P, rows, D):
    rng = np.random.default_rng(P * 1000 + rows)
    o = rng.standard_normal((P, rows, D)).astype(np.float32)
    lse = (rng.standard_normal((P, rows)) * 3).astype(np.float32)
    empty = rng.random((P, rows)) < 0.3
    lse[empty] = -np.inf
    o[empty] = np.nan                      # an empty part's O must not be read
    lse[:, : min(3, rows)] = -np.inf       # rows with no allowed key at all
    o_out, lse_out = cp.merge_partials(torch.from_numpy(o).cuda(), torch.from_numpy(lse).cuda())
    o_ref, l_ref = A.merge([(np.where(np.isnan(o[t]), 0, o[t]), lse[t]) for t in range(P)])
    o_gpu = o_out.double().cpu().numpy()
    l_gpu = lse_out.double().cpu().numpy()
    fin = np.isfinite(l_ref)
    assert np.array_equal(np.isfinite(l_gpu), fin)
    assert np.all(o_gpu[~fin] == 0)
    d = np.abs(o_gpu - o_ref)
    assert d.max() <= G.TOL_O_MAX and d.mean() <= G.TOL_O_MEAN
    assert np.abs(l_gpu[fin] - l_ref[fin]).max() <= 1e-4


@pytest.mark.parametrize("B,H,S,D,N,layout", [(1, 2, 1024, 128, 4, "zigzag"), (2, 2, 800, 64, 4, "contiguous"),
                                              (1, 3, 384, 128, 3, "zigzag")])
def test_partials_match_oracle_ring_steps(B, H, S, D, N, layout):
    q, k, v = make_small(B, H, S, D, 40 + N)
    plan = cp.Plan(B, H, S, D, N, True, layout)
    qd, kd, vd = (G.to_layout(x, N, layout).cuda() for x in (q, k, v))
    op, lp = cp.attn_fwd_partials(plan, qd, kd, vd)
    assert cp.check(plan) == 0
    f = lambda t: t.float().numpy()
    parts = A.ring_partials(f(q), f(k), f(v), L.rank_major_map(B, S, N, layout), N, causal=True)
    T = S // N
    op = op.double().cpu().numpy().reshape(N, N, B, T, H, D)      # [step][rank][b][tl][h][d]
    lp = lp.double().cpu().numpy().reshape(N, N, B, T, H)
    for r in range(N):
        for t in range(N):
            o_ref = parts[r][t][0]                   # [B, T, H, D]
            l_ref = parts[r][t][1].transpose(0, 2, 1)  # [B, T, H]
            fin = np.isfinite(l_ref)
            assert np.array_equal(np.isfinite(lp[t, r]), fin), (r, t)
            assert np.all(op[t, r][~fin] == 0)
            d = np.abs(op[t, r] - o_ref)
            assert d.max() <= G.TOL_O_MAX and d.mean() <= G.TOL_O_MEAN, (r, t, d.max())
            if fin.any():
                assert np.abs(lp[t, r][fin] - l_ref[fin]).max() <= G.TOL_LSE


def test_partials_plus_merge_equals_fused():
    w = WORKLOADS["zigzag_4k"]
    q, k, v = make_qkv(w)
    plan = cp.Plan(w.B, w.H, w.S, w.D, w.N, w.causal, w.layout)
    qd, kd, vd = (G.to_layout(x, w.N, w.layout).cuda() for x in (q, k, v))
    o_f, lse_f = cp.attn_fwd(plan, qd, kd, vd)
    op, lp = cp.attn_fwd_partials(plan, qd, kd, vd)
    o_m, lse_m = cp.merge_partials(op, lp)
    assert cp.check(plan) == 0
    d = (o_m.float().reshape(o_f.shape) - o_f.float()).abs()
    assert d.max().item() <= G.TOL_O_MAX and d.mean().item() <= G.TOL_O_MEAN
    # lse_m is in row order [N][B][T][H]; bring it to natural [B][H][S]
    T = w.S // w.N
    m = torch.from_numpy(G.token_map(w.B, w.S, w.N, w.layout))
    lm = lse_m.cpu().reshape(w.N * w.B * T, w.H)
    nat = torch.empty(w.B * w.S, w.H)
    nat[m] = lm
    nat = nat.reshape(w.B, w.S, w.H).permute(0, 2, 1)
    assert (nat - lse_f.cpu()).abs().max().item() <= G.TOL_LSE


def test_ulysses_partials_unsupported():
    plan = cp.Plan(1, 8, 512, 128, 4, False, "ulysses")
    x = torch.zeros(4, 1, 128, 8, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cp.CpAttnError) as e:
        cp.attn_fwd_partials(plan, x, x, x)
    assert e.value.status == -2
