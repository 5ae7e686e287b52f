"""GPU checks of the ring's rank-local path against the oracle.

* ``cp_attn_fwd_ring_step``: every (rank, step) partial, computed from rank-local
  buffers, against the oracle's ring partial of that rank and step;
* ``cp_attn_fwd_ring`` (a rank's N steps in one cooperative launch): bit-identical
  to the N per-step launches (the same unit arithmetic), both on resident blocks
  and when its copy warps fetch the other blocks themselves (the fetched slots
  bit-identical to their sources); an arrival count that never fills ends the
  kernel with CP_ERR_TIMEOUT and leaves the context usable;
* the whole ring (``ring.RingRank``): N ranks emulated as host threads of one
  process on one GPU (their launches on one stream), one host barrier per call,
  calls back to back; each rank's rows against the oracle's full attention, and
  against the fused single-launch forward on the 4k zigzag workload;
* the IPC plumbing that can run in one process (handles, device views).
The rank processes of a real multi-GPU ring need one GPU each; their protocol is
checked on CPU with gloo processes (tests/test_ring_host.py).
"""
import numpy as np
import pytest
import torch

import context_long_sequence_cp_b200 as cp
from context_long_sequence_cp_b200 import ring as R
from oracle import attention as A
from oracle import layouts as L
from tests import gpu_util as G
from workloads import WORKLOADS, make_qkv, make_small

pytestmark = pytest.mark.gpu


def _rank_inputs(x, N, layout):
    """natural [B, S, H, D] -> per-rank contiguous [B, S/N, H, D] tensors on the GPU."""
    y = G.to_layout(x, N, layout).cuda()
    return [y[r].contiguous() for r in range(N)]


@pytest.mark.parametrize("B,H,S,D,N,layout,causal", [
    (1, 2, 256, 64, 4, "contiguous", False),
    (1, 2, 1024, 128, 4, "zigzag", True),
    (2, 2, 1536, 64, 3, "contiguous", True),
    (1, 3, 1920, 128, 5, "zigzag", True),      # 384 local tokens: a ragged query-tile pair
])
def test_ring_step_matches_oracle_partials(B, H, S, D, N, layout, causal):
    q, k, v = make_small(B, H, S, D, 60 + N)
    plan = cp.Plan(B, H, S, D, N, causal, layout)
    qs, ks, vs = (_rank_inputs(x, N, layout) for x in (q, k, v))
    f = lambda t: t.float().numpy()
    parts = A.ring_partials(f(q), f(k), f(v), L.rank_major_map(B, S, N, layout), N, causal=causal)
    T = S // N
    for r in range(N):
        for t in range(N):
            rk = (r + t) % N
            op, lp = cp.attn_fwd_ring_step(plan, r, t, qs[r], ks[rk], vs[rk])
            assert cp.check(plan) == 0
            op = op.double().cpu().numpy().reshape(B, T, H, D)
            lp = lp.double().cpu().numpy().reshape(B, T, H)
            o_ref = parts[r][t][0]
            l_ref = parts[r][t][1].transpose(0, 2, 1)
            fin = np.isfinite(l_ref)
            assert np.array_equal(np.isfinite(lp), fin), (r, t)
            assert np.all(op[~fin] == 0)
            d = np.abs(op - o_ref)
            assert d.max() <= G.TOL_O_MAX and d.mean() <= G.TOL_O_MEAN, (r, t, d.max())
            if fin.any():
                assert np.abs(lp[fin] - l_ref[fin]).max() <= G.TOL_LSE


@pytest.mark.parametrize("B,H,S,D,N,layout,causal", [
    (1, 2, 1024, 128, 4, "zigzag", True),
    (2, 2, 1536, 64, 3, "contiguous", True),
    (1, 3, 1920, 128, 5, "zigzag", True),
    (1, 2, 4096, 128, 8, "zigzag", True),
    (1, 2, 512, 64, 2, "contiguous", False),
])
def test_ring_launch_equals_step_launches(B, H, S, D, N, layout, causal):
    q, k, v = make_small(B, H, S, D, 80 + N)
    plan = cp.Plan(B, H, S, D, N, causal, layout)
    qd, kd, vd = (G.to_layout(x, N, layout).cuda() for x in (q, k, v))
    split = N if N <= 2 else (N + 1) // 2
    assert plan.ring_parts() == (split + 1 if split < N else N)
    f = lambda t: t.float().numpy()
    parts = A.ring_partials(f(q), f(k), f(v), L.rank_major_map(B, S, N, layout), N, causal=causal)
    T = S // N
    arrived = torch.zeros(N, dtype=torch.int32, device="cuda")
    for r in range(N):
        op, lp = cp.attn_fwd_ring(plan, r, qd[r], kd, vd)                  # every block resident
        # fused pull: only the own slot is filled; the copy warps fetch the rest
        ks = torch.full_like(kd, float("nan"))
        vs = torch.full_like(vd, float("nan"))
        ks[r].copy_(kd[r])
        vs[r].copy_(vd[r])
        srcs_k = [kd[j].data_ptr() for j in range(N)]
        srcs_v = [vd[j].data_ptr() for j in range(N)]
        op2, lp2 = cp.attn_fwd_ring(plan, r, qd[r], ks, vs, srcs_k, srcs_v, arrived)
        assert cp.check(plan) == 0
        assert torch.equal(ks.view(torch.int16), kd.view(torch.int16))
        assert torch.equal(vs.view(torch.int16), vd.view(torch.int16))
        if N > 1:
            chunks = -(-kd[0].numel() * 2 // 32768)
            assert arrived.tolist() == [0 if j == r else 2 * chunks for j in range(N)]
        assert torch.equal(op.view(torch.int32), op2.view(torch.int32))
        assert torch.equal(lp.view(torch.int32), lp2.view(torch.int32))
        for t in range(split):               # first phase: the per-step partials, bit for bit
            rk = (r + t) % N
            os_, ls_ = cp.attn_fwd_ring_step(plan, r, t, qd[r], kd[rk].contiguous(), vd[rk].contiguous())
            assert torch.equal(op[t].view(torch.int32), os_.view(torch.int32)), (r, t)
            assert torch.equal(lp[t].view(torch.int32), ls_.view(torch.int32)), (r, t)
        if split < N:                        # tail: the merge of steps split..N-1 (oracle)
            o_ref, l_ref = A.merge([(parts[r][t][0].reshape(-1, D),
                                     parts[r][t][1].transpose(0, 2, 1).reshape(-1)) for t in range(split, N)])
            o_t = op[split].double().cpu().numpy()
            l_t = lp[split].double().cpu().numpy()
            fin = np.isfinite(l_ref)
            assert np.array_equal(np.isfinite(l_t), fin)
            d = np.abs(o_t - o_ref)
            assert d.max() <= G.TOL_O_MAX and d.mean() <= G.TOL_O_MEAN, (r, d.max())
            if fin.any():
                assert np.abs(l_t[fin] - l_ref[fin]).max() <= G.TOL_LSE
    assert cp.check(plan) == 0


def test_ring_launch_times_out_on_a_block_that_never_arrives():
    B, H, S, D, N = 1, 2, 1024, 128, 4
    q, k, v = make_small(B, H, S, D, 90)
    plan = cp.Plan(B, H, S, D, N, True, "zigzag")
    qd, kd, vd = (G.to_layout(x, N, "zigzag").cuda() for x in (q, k, v))
    arrived = torch.zeros(N, dtype=torch.int32, device="cuda")     # nothing raises the counts
    cp.attn_fwd_ring_external(plan, 0, qd[0], kd, vd, arrived)
    assert cp.check(plan) == -5                                    # CP_ERR_TIMEOUT, after the 2 s budget
    assert cp.check(plan) == 0
    # the context is still usable: the same launch with the blocks marked arrived
    arrived.fill_(1)
    op, lp = cp.attn_fwd_ring_external(plan, 0, qd[0], kd, vd, arrived)
    assert cp.check(plan) == 0
    os_, ls_ = cp.attn_fwd_ring_step(plan, 0, 1, qd[0], kd[1].contiguous(), vd[1].contiguous())
    assert torch.equal(op[1].view(torch.int32), os_.view(torch.int32))


def _run_ring(plan, qs, ks, vs, reps=1):
    ranks = R.thread_ring(plan)
    try:
        outs = []
        for _ in range(reps):
            out = R.run_threads(ranks, list(zip(qs, ks, vs)))
            outs.append([(o.clone(), l.clone()) for o, l in out])
        torch.cuda.synchronize()
        assert cp.check(plan) == 0
        return outs[-1]
    finally:
        for rr in ranks:
            rr.close()


@pytest.mark.parametrize("B,H,S,D,N,layout,causal", [
    (1, 2, 256, 64, 4, "contiguous", False),
    (1, 2, 2048, 128, 4, "zigzag", True),
    (2, 2, 1536, 64, 3, "contiguous", True),
    (1, 2, 1024, 128, 2, "zigzag", True),
    (1, 2, 512, 128, 1, "contiguous", True),
])
def test_ring_threads_match_oracle(B, H, S, D, N, layout, causal):
    q, k, v = make_small(B, H, S, D, 70 + N)
    plan = cp.Plan(B, H, S, D, N, causal, layout)
    qs, ks, vs = (_rank_inputs(x, N, layout) for x in (q, k, v))
    out = _run_ring(plan, qs, ks, vs, reps=3)       # calls alternate between the two slot sets
    f = lambda t: t.float().numpy()
    o_ref, lse_ref = A.attention(f(q), f(k), f(v), causal=causal)       # [B, S, H, D], [B, H, S]
    pos = L.chunk_positions(S, N, layout)
    T = S // N
    for r in range(N):
        o, lse = out[r]
        o = o.double().cpu().numpy()                                     # [B, T, H, D]
        lse = lse.double().cpu().numpy().reshape(B, T, H)
        d = np.abs(o - o_ref[:, pos[r]])
        assert d.max() <= G.TOL_O_MAX and d.mean() <= G.TOL_O_MEAN, (r, d.max())
        assert np.abs(lse - lse_ref[:, :, pos[r]].transpose(0, 2, 1)).max() <= G.TOL_LSE


def test_ring_threads_match_fused_zigzag_4k():
    w = WORKLOADS["zigzag_4k"]
    q, k, v = make_qkv(w)
    plan = cp.Plan(w.B, w.H, w.S, w.D, w.N, w.causal, w.layout)
    qd, kd, vd = (G.to_layout(x, w.N, w.layout).cuda() for x in (q, k, v))
    o_f, lse_f = cp.attn_fwd(plan, qd, kd, vd)
    out = _run_ring(plan, [qd[r].contiguous() for r in range(w.N)], [kd[r].contiguous() for r in range(w.N)],
                    [vd[r].contiguous() for r in range(w.N)])
    T = w.S // w.N
    pos = L.chunk_positions(w.S, w.N, w.layout)
    for r in range(w.N):
        o, lse = out[r]
        d = (o.float() - o_f[r].float()).abs()
        assert d.max().item() <= G.TOL_O_MAX and d.mean().item() <= G.TOL_O_MEAN
        l_f = lse_f[:, :, torch.from_numpy(pos[r]).cuda()].permute(0, 2, 1)      # [B, T, H]
        assert (lse.reshape(w.B, T, w.H) - l_f).abs().max().item() <= G.TOL_LSE
    # sampled rows of rank 0 and the last rank against the oracle too
    rows = np.array([[0, h, int(p)] for h in (0, w.H - 1) for p in (pos[0, 5], pos[0, -1], pos[-1, 7], pos[-1, -3])])
    o_ref, l_ref = G.oracle_rows(q, k, v, rows, w.causal)
    o_nat = G.from_layout(torch.stack([o for o, _ in out]), w.N, w.layout)
    ix = [torch.from_numpy(rows[:, j]).cuda() for j in (0, 2, 1)]
    got = o_nat[ix[0], ix[1], ix[2]].double().cpu().numpy()
    assert np.abs(got - o_ref).max() <= G.TOL_O_MAX


def test_ring_buffers_and_ipc_handle():
    buf = cp.DeviceBuffer(1 << 20)
    try:
        h = buf.ipc_handle()
        assert len(h) == 64 and any(h)
        t = buf.view((512, 1024), torch.bfloat16, device="cuda")
        t.copy_(torch.arange(512 * 1024, device="cuda").reshape(512, 1024).to(torch.bfloat16))
        dst = torch.empty(512, 1024, dtype=torch.bfloat16, device="cuda")
        cp.copy_async(dst.data_ptr(), buf.ptr, 1 << 20)
        torch.cuda.synchronize()
        assert torch.equal(dst.view(torch.int16), t.view(torch.int16))
    finally:
        buf.close()


def test_ring_step_rejects_bad_arguments():
    plan = cp.Plan(1, 2, 1024, 64, 4, True, "zigzag")
    x = torch.zeros(1, 256, 2, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cp.CpAttnError) as e:
        cp.attn_fwd_ring_step(plan, 4, 0, x, x, x)
    assert e.value.status == -1
    with pytest.raises(cp.CpAttnError) as e:
        cp.attn_fwd_ring_step(plan, 0, 0, x.view(-1)[1:], x, x)      # 2 bytes past a 16-byte boundary
    assert e.value.status == -3


@pytest.mark.parametrize("name,layout,rank", [("zigzag_32k", "zigzag", 3), ("long_128k", "contiguous", 2),
                                              ("long_128k", "zigzag", 1)])
def test_ring_rank_full_size_sampled_rows(name, layout, rank):
    """One rank of a full-size workload, as bench.py runs it: one cooperative
    launch fetching the other ranks' blocks, then the merge; the rank's rows among
    the workload's sampled rows against the oracle."""
    from workloads import sample_rows
    w = WORKLOADS[name]
    q, k, v = make_qkv(w)
    N, T = w.N, w.S // w.N
    plan = cp.Plan(w.B, w.H, w.S, w.D, N, w.causal, layout)
    qd, kd, vd = (G.to_layout(x, N, layout).cuda() for x in (q, k, v))
    ks, vs = torch.empty_like(kd), torch.empty_like(vd)
    ks[rank].copy_(kd[rank])
    vs[rank].copy_(vd[rank])
    arrived = torch.zeros(N, dtype=torch.int32, device="cuda")
    op, lp = cp.attn_fwd_ring(plan, rank, qd[rank], ks, vs, [kd[j].data_ptr() for j in range(N)],
                              [vd[j].data_ptr() for j in range(N)], arrived)
    o, lse = cp.merge_partials(op, lp)
    assert cp.check(plan) == 0
    del ks, vs, op, lp
    pos = L.chunk_positions(w.S, N, layout)[rank]
    local = {int(p): i for i, p in enumerate(pos)}
    rows = np.array([r for r in sample_rows(w) if int(r[2]) in local])[:256]
    assert len(rows) > 16
    o_ref, l_ref = G.oracle_rows(q, k, v, rows, w.causal)
    ix = torch.from_numpy(np.array([(r[0] * T + local[int(r[2])]) * w.H + r[1] for r in rows])).cuda()
    got = o[ix].double().cpu().numpy()
    got_l = lse[ix].double().cpu().numpy()
    d = np.abs(got - o_ref)
    assert d.max() <= G.TOL_O_MAX and d.mean() <= G.TOL_O_MEAN, d.max()
    assert np.abs(got_l - l_ref).max() <= G.TOL_LSE
