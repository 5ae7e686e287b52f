"""GPU parity of the sequence-parallel step (cp_sp_rs_dropout_add_ln) against the
fp64 oracle: z = dropout(sum of partials) + residual, y = LayerNorm(z).

Tolerances, from the arithmetic: the kernel sums bf16 partials in fp32 and rounds z
to bf16 once (at most one ulp, 2^-8 relative, plus the fp32 sum's ~1e-6 of the
summed magnitudes); y is computed from the fp32 z (not the rounded one) and
rounded once: |y - oracle| <= 2^-8 |oracle| + 2e-3. The dropout decision is the
given mask, so dropped elements are exactly the residual (or exactly 0).
"""
import numpy as np
import pytest
import torch

import context_long_sequence_cp_b200 as cp
from oracle import sp_norm as SP
from workloads import make_keep_bits

pytestmark = pytest.mark.gpu


def _inputs(nparts, rows, H, seed, residual=True):
    g = torch.Generator().manual_seed(seed)
    parts = torch.randn(nparts, rows, H, generator=g).to(torch.bfloat16)
    res = torch.randn(rows, H, generator=g).to(torch.bfloat16) if residual else None
    gamma = (1.0 + 0.1 * torch.randn(H, generator=g)).float()
    beta = (0.1 * torch.randn(H, generator=g)).float()
    return parts, res, gamma, beta


@pytest.mark.parametrize("nparts,rows,H,p,residual", [
    (2, 64, 256, 0.1, True),
    (8, 2048, 4096, 0.1, True),      # 8 tensor-parallel ranks, 7B-like hidden size
    (1, 37, 8192, 0.0, False),       # largest H, odd row count, LayerNorm only
    (3, 6, 8, 0.5, True),            # smallest H: one vector per row
    (4, 300, 1024, 0.3, False),
])
def test_sp_step_matches_oracle(nparts, rows, H, p, residual):
    parts, res, gamma, beta = _inputs(nparts, rows, H, seed=rows + H)
    keep, bits = make_keep_bits(rows, H, p, seed=H) if p > 0 else (None, None)
    z, y = cp.sp_rs_dropout_add_ln(parts.cuda(), bits.cuda() if bits is not None else None, p,
                                   res.cuda() if res is not None else None, gamma.cuda(), beta.cuda())
    torch.cuda.synchronize()
    z_ref, y_ref = SP.rs_dropout_add_ln(parts.float().numpy(), keep, p,
                                        res.float().numpy() if res is not None else None,
                                        gamma.numpy(), beta.numpy())
    zg, yg = z.double().cpu().numpy(), y.double().cpu().numpy()
    mag = np.abs(parts.float().numpy()).sum(0) / (1 - p) + (np.abs(res.float().numpy()) if res is not None else 0)
    assert np.all(np.abs(zg - z_ref) <= 2.0 ** -8 * np.abs(z_ref) + 1e-6 * mag + 1e-30)
    assert np.all(np.abs(yg - y_ref) <= 2.0 ** -8 * np.abs(y_ref) + 2e-3)
    if keep is not None:
        dropped = ~keep
        want = res.float().numpy()[dropped] if res is not None else 0.0
        assert np.array_equal(zg[dropped], np.broadcast_to(want, zg[dropped].shape))


def test_sp_step_single_outputs_and_shard_concat():
    # z only, then y only; and the pages' check on the GPU side: LayerNorm of the
    # rows of each of N shards, computed shard by shard, equals the whole at once.
    nparts, rows, H, N = 2, 96, 512, 3
    parts, res, gamma, beta = _inputs(nparts, rows, H, seed=7)
    z_only, y_none = cp.sp_rs_dropout_add_ln(parts.cuda(), residual=res.cuda(), want_y=False)
    assert y_none is None
    z_none, y_only = cp.sp_rs_dropout_add_ln(parts.cuda(), residual=res.cuda(), gamma=gamma.cuda(),
                                             beta=beta.cuda(), want_z=False)
    assert z_none is None
    z_all, y_all = cp.sp_rs_dropout_add_ln(parts.cuda(), residual=res.cuda(), gamma=gamma.cuda(), beta=beta.cuda())
    assert torch.equal(z_only, z_all) and torch.equal(y_only, y_all)
    shard = rows // N
    ys = [cp.sp_rs_dropout_add_ln(parts[:, i * shard:(i + 1) * shard].contiguous().cuda(),
                                  residual=res[i * shard:(i + 1) * shard].contiguous().cuda(),
                                  gamma=gamma.cuda(), beta=beta.cuda())[1] for i in range(N)]
    assert torch.equal(torch.cat(ys, 0), y_all)
