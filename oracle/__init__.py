"""CPU fp64 oracle for context-parallel attention — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may import anything from this package. The product path (the
CUDA library under ``context_long_sequence_cp_b200/`` and its binding) never
imports, links or calls it, and shares no code with it: the only common module
is ``workloads``, which makes seeded inputs and holds none of the method's
arithmetic.

Contents:
  * ``attention``  — softmax attention with per-row logsumexp, by definition
    (matrix form and a brute-force row loop), the partial result of a query
    block against one key/value chunk, and the logsumexp-weighted merge of
    partials.
  * ``layouts``    — the contiguous / zigzag rank-major token maps and the
    Ulysses sequence-shard <-> head-group run maps, as int64 index arrays.
  * ``schedule``   — brute-force (query tile, key tile) pair classification and
    per-rank executed tile counts.
  * ``rope``       — rotary position embedding at global positions.
  * ``attention_bwd`` — gradients of softmax attention (dQ, dK, dV), by the
    chain rule on the forward's definition.
  * ``sp_norm``    — reduce-scatter / all-gather over virtual ranks and the
    LayerNorm + dropout + residual step on sequence shards.

Every function is pinned by ``tests/test_oracle_*.py`` against something other
than itself (library special cases, closed forms, invariants, hand-derived
worked examples under ``tests/golden/``). No function here is "parity
unpinned".
"""
from . import attention, attention_bwd, layouts, rope, schedule, sp_norm  # noqa: F401
