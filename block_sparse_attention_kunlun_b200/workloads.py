"""Seeded synthetic inputs for block attention.

This module only draws random numbers and builds the rotary tables a
caller supplies; it holds none of the attention arithmetic, so both the CUDA
path and the CPU oracle can be fed from it.

The pages describe the workload only in words: user-engagement histories
whose lengths run from hundreds to tens of thousands of events, batched as
jagged tensors without padding ("GEM (Meta)", section "Training
infrastructure"). The five shapes below stand in for that workload; they
name no dataset and none exists to stand in for.

Recipe (every config): one ``torch.Generator`` on the CPU seeded with
``1000 + config``; draws in a fixed order -- example lengths, skip flags,
q, k, v, dout -- each as float32 ``randn`` (lengths as integers, skip flags
as uniform [0, 1) compared with the skip probability); q, k, v are
multiplied by ``qkv_scale`` and the tensors are cast to the config dtype.
Layout: q, k, v, dout are ``[total_tokens, heads, head_dim]``; seq_offsets
is int32 ``[batch + 1]`` (prefix sums of the lengths); skip is uint8
``[batch]`` or None.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: torch.dtype
    batch: int
    len_lo: int          # lengths are drawn uniformly from [len_lo, len_hi] (inclusive)
    len_hi: int
    heads: int
    head_dim: int
    block: int
    window: int
    qkv_scale: float
    fwd_only: bool = False
    skip_p: float = 0.0
    seed: int = 0

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads, numbered as in the project's scope table.
CONFIGS = {
    1: Workload("fp32 fwd, 2 x 256, H2 D32, block 64, window 1", torch.float32,
                2, 256, 256, 2, 32, 64, 1, 1.0, fwd_only=True, seed=1001),
    2: Workload("bf16, 64 x 1024, H4 D64, block 128, window 2", torch.bfloat16,
                64, 1024, 1024, 4, 64, 128, 2, 1.0 / math.sqrt(64), seed=1002),
    3: Workload("bf16 jagged, 256 x U[64,4096], H8 D128, block 256, window 2", torch.bfloat16,
                256, 64, 4096, 8, 128, 256, 2, 1.0 / math.sqrt(128), seed=1003),
    4: Workload("bf16, 8 x 32768, H8 D128, block 512, window 4", torch.bfloat16,
                8, 32768, 32768, 8, 128, 512, 4, 1.0 / math.sqrt(128), seed=1004),
    5: Workload("bf16 jagged + skip p=0.43, 256 x U[64,4096], H8 D128, block 256, window 2",
                torch.bfloat16, 256, 64, 4096, 8, 128, 256, 2, 1.0 / math.sqrt(128),
                skip_p=0.43, seed=1005),
}


def draw_lengths(w: Workload, gen: torch.Generator) -> torch.Tensor:
    if w.len_lo == w.len_hi:
        return torch.full((w.batch,), w.len_lo, dtype=torch.int64)
    return torch.randint(w.len_lo, w.len_hi + 1, (w.batch,), generator=gen, dtype=torch.int64)


def make_inputs(w: Workload, seed: int | None = None, q_gain: float = 1.0,
                lengths: list[int] | None = None, want_dout: bool | None = None) -> dict:
    """Draw one batch for workload ``w`` on the CPU.

    ``q_gain`` multiplies q after the config scaling (peaked-softmax stress
    cases); ``lengths`` overrides the drawn lengths (the draw still happens so
    later draws stay aligned). Returns a dict of CPU tensors.
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(w.seed if seed is None else seed)
    lens = draw_lengths(w, gen)
    if lengths is not None:
        lens = torch.tensor(lengths, dtype=torch.int64)
    batch = lens.shape[0]
    skip_u = torch.rand((w.batch,), generator=gen)
    skip = None
    if w.skip_p > 0.0:
        skip = (skip_u[:batch] < w.skip_p).to(torch.uint8)
        if skip.shape[0] < batch:
            raise ValueError("more lengths than the workload's batch")
    offs = torch.zeros(batch + 1, dtype=torch.int64)
    offs[1:] = torch.cumsum(lens, 0)
    T = int(offs[-1])
    shape = (T, w.heads, w.head_dim)

    def normal(scale):
        x = torch.randn(shape, generator=gen, dtype=torch.float32)
        if scale != 1.0:
            x.mul_(scale)
        return x.to(w.dtype)

    q = normal(w.qkv_scale * q_gain)
    k = normal(w.qkv_scale)
    v = normal(w.qkv_scale)
    out = dict(seq_offsets=offs.to(torch.int32), q=q, k=k, v=v, skip=skip,
               lengths=lens, workload=w)
    if want_dout if want_dout is not None else not w.fwd_only:
        out["dout"] = normal(1.0)
    return out


def rope_tables(rows: int, head_dim: int, base: float = 10000.0):
    """cos and sin tables, float32 [rows, head_dim / 2], for rotary position
    embeddings with RoFormer's frequencies: entry [p, k] is the cosine (sine)
    of p * base ** (-2k / head_dim). Angles are formed in float64 and the
    results rounded to float32 (the tables the library reads)."""
    p = torch.arange(rows, dtype=torch.float64)[:, None]
    inv_freq = base ** (-2.0 * torch.arange(head_dim // 2, dtype=torch.float64) / head_dim)
    ang = p * inv_freq[None, :]
    return torch.cos(ang).to(torch.float32), torch.sin(ang).to(torch.float32)
