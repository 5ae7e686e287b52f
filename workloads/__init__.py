"""Seeded synthetic workloads for context-parallel attention.

This module holds the five workload shapes, their seeds and value scales, the
seeded Q/K/V generators and the seeded choice of sampled query rows. It holds
none of the attention arithmetic: both the CPU oracle (``oracle/``) and the GPU
path's tests and benchmark draw their inputs from here, so the two sides see
bit-identical bf16 inputs.

Generation recipe (one per workload):
  * ``torch.Generator('cpu').manual_seed(seed)``;
  * Q, then K, then V drawn with ``torch.randn`` in fp32, natural layout
    ``[B, S, H, D]`` (batch, token, head, head dim);
  * each multiplied by its scale (0.5 for Q and K of the 32k workload; exact in
    fp32), then rounded to bf16 (round-to-nearest-even).
The Ulysses workload's sequence shards are the natural tensor split along S into
N equal pieces, i.e. the contiguous rank-major layout ``[N, B, S/N, H, D]``.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    S: int
    D: int
    N: int
    causal: bool
    layout: str            # "contiguous" | "zigzag" | "ulysses"
    seed: int
    q_scale: float = 1.0
    k_scale: float = 1.0
    v_scale: float = 1.0
    sample_rows: Optional[int] = None   # None: compare every row
    # A second layout over the same inputs whose output must agree (long context).
    alt_layout: Optional[str] = None

    @property
    def flops(self) -> float:
        """Counted FLOPs: 4*B*H*S^2*D, halved when causal."""
        f = 4.0 * self.B * self.H * self.S * self.S * self.D
        return f / 2 if self.causal else f

    def with_layout(self, layout: str) -> "Workload":
        return dataclasses.replace(self, layout=layout, alt_layout=None)


WORKLOADS = {
    # B1 H2 S256 D64, 4 virtual ranks of 64-token chunks, non-causal, contiguous.
    "tiny": Workload("tiny", B=1, H=2, S=256, D=64, N=4, causal=False,
                     layout="contiguous", seed=0),
    # B1 H16 S4096 D128, 4 ranks, causal, zigzag (512-token chunks).
    "zigzag_4k": Workload("zigzag_4k", B=1, H=16, S=4096, D=128, N=4, causal=True,
                          layout="zigzag", seed=1),
    # 7B-shaped: B1 H32 S32768 D128, 8 ranks, causal, zigzag; Q,K scaled by 0.5.
    "zigzag_32k": Workload("zigzag_32k", B=1, H=32, S=32768, D=128, N=8, causal=True,
                           layout="zigzag", seed=2, q_scale=0.5, k_scale=0.5,
                           sample_rows=4096),
    # 128k long context: B1 H32 S131072 D128, 4 ranks, causal, contiguous vs zigzag.
    "long_128k": Workload("long_128k", B=1, H=32, S=131072, D=128, N=4, causal=True,
                          layout="contiguous", seed=3, sample_rows=4096,
                          alt_layout="zigzag"),
    # Ulysses head-sharded: B2 S16384 H32 D128, 8 ranks, 4 heads per group, non-causal.
    "ulysses_16k": Workload("ulysses_16k", B=2, H=32, S=16384, D=128, N=8, causal=False,
                            layout="ulysses", seed=4, sample_rows=4096),
}


def make_qkv(w: Workload, device: str = "cpu"):
    """Seeded bf16 Q, K, V in natural layout [B, S, H, D]."""
    g = torch.Generator("cpu")
    g.manual_seed(w.seed)
    out = []
    for scale in (w.q_scale, w.k_scale, w.v_scale):
        x = torch.randn(w.B, w.S, w.H, w.D, generator=g, dtype=torch.float32)
        if scale != 1.0:
            x.mul_(scale)
        out.append(x.to(torch.bfloat16).to(device))
    return tuple(out)


def make_small(B, H, S, D, seed, scale=1.0, device="cpu"):
    """Seeded bf16 Q, K, V of an arbitrary small shape (edge-case tests)."""
    g = torch.Generator("cpu")
    g.manual_seed(seed)
    out = []
    for _ in range(3):
        x = torch.randn(B, S, H, D, generator=g, dtype=torch.float32) * scale
        out.append(x.to(torch.bfloat16).to(device))
    return tuple(out)


def make_dout(shape, seed):
    """Seeded upstream gradient dO for the backward: randn fp32 -> bf16, drawn
    from its own generator (seed 1000 + seed) in natural [B, S, H, D] order."""
    g = torch.Generator("cpu")
    g.manual_seed(1000 + seed)
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def make_keep_bits(rows: int, H: int, p: float, seed: int):
    """Dropout keep mask (the random draw of dropout) for rows x H elements: keep
    where a seeded uniform draw exceeds p, as the 5688vip.com page's dropout does.
    Returns (keep bool [rows, H], packed int32 [ceil(rows*H/32)]: bit i % 32 of word
    i/32 holds flat element i; unused bits of the last word are 0)."""
    g = torch.Generator("cpu")
    g.manual_seed(2000 + seed)
    keep = torch.rand(rows, H, generator=g) > p
    packed = np.packbits(keep.numpy().reshape(-1), bitorder="little")
    packed = np.concatenate([packed, np.zeros((-len(packed)) % 4, dtype=np.uint8)]).view(np.int32)
    return keep.numpy(), torch.from_numpy(packed.copy())


def sample_rows(w: Workload, n: Optional[int] = None) -> np.ndarray:
    """Sampled query rows (b, h, i) in natural coordinates, int64 [n_rows, 3].

    Rows are drawn uniformly without replacement with
    ``np.random.default_rng(10_000 + seed)``; to them are added row 0, row S-1
    and the first and last row of every chunk of length S/(2N) (which covers
    the chunk edges of both the contiguous and the zigzag split) at b=0, h=0.
    With ``sample_rows`` unset every row is returned.
    """
    n = w.sample_rows if n is None else n
    if n is None:
        b, h, i = np.meshgrid(np.arange(w.B), np.arange(w.H), np.arange(w.S), indexing="ij")
        return np.stack([b.ravel(), h.ravel(), i.ravel()], axis=1).astype(np.int64)
    rng = np.random.default_rng(10_000 + w.seed)
    total = w.B * w.H * w.S
    flat = rng.choice(total, size=min(n, total), replace=False)
    rows = set(int(x) for x in flat)
    c = w.S // (2 * w.N)
    forced = {0, w.S - 1}
    for k in range(2 * w.N):
        forced.add(k * c)
        forced.add(k * c + c - 1)
    for i in forced:
        rows.add(i)   # b=0, h=0 -> flat index i
    rows = np.array(sorted(rows), dtype=np.int64)
    b = rows // (w.H * w.S)
    h = (rows // w.S) % w.H
    i = rows % w.S
    return np.stack([b, h, i], axis=1)
