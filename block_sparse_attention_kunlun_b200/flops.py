"""Work accounting for block attention (host-side, used by the benchmark).

Useful work is counted only inside the mask: a query at local index i sees
i - window_start(i) + 1 keys, window_start(i) = max(0, (i // block -
(window - 1)) * block). Per visible (query, key) pair and head:
  forward  4 D FLOPs (q.k and p*v),
  backward 10 D FLOPs (S recomputed from lse, dP, dV, dK, dQ),
so a training step costs 14 D FLOPs per pair. Skipped and empty examples
count nothing.

Algorithmic bytes (each tensor touched once, bf16 = 2 bytes, fp32 = 4):
  forward  reads q, k, v; writes out, lse;
  backward reads q, k, v, out, dout, lse; writes dq, dk, dv.
"""
from __future__ import annotations

import numpy as np


def visible_pairs(lengths, block: int, window: int, skip=None) -> int:
    """Number of visible (query, key) pairs per head, summed over examples."""
    total = 0
    for e, L in enumerate(np.asarray(lengths, dtype=np.int64)):
        if L <= 0 or (skip is not None and skip[e]):
            continue
        i = np.arange(L, dtype=np.int64)
        ws = np.maximum(0, (i // block - (window - 1)) * block)
        total += int(np.sum(i - ws + 1))
    return total


def live_tokens(lengths, skip=None) -> int:
    lengths = np.asarray(lengths, dtype=np.int64)
    if skip is None:
        return int(lengths.sum())
    return int(lengths[np.asarray(skip) == 0].sum())


def step_flops(pairs: int, heads: int, head_dim: int) -> dict:
    """Useful FLOPs of one forward, one backward, and one training step."""
    f = 4 * head_dim * pairs * heads
    b = 10 * head_dim * pairs * heads
    return {"fwd": f, "bwd": b, "step": f + b}


def step_bytes(total_tokens: int, heads: int, head_dim: int, elem_bytes: int = 2) -> dict:
    """Algorithmic HBM bytes of one forward and one backward."""
    t = total_tokens * heads * head_dim * elem_bytes
    lse = total_tokens * heads * 4
    return {"fwd": 3 * t + t + lse, "bwd": 5 * t + lse + lse + 3 * t}
