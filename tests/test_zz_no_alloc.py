"""The forward entry point that allocates nothing (ba_fwd_noalloc).

It exists for callers that cannot allocate device memory: a serving loop
recording its forward into a CUDA graph (no allocation during stream
capture) or a framework that owns all device memory. Its scratch is a fixed
array inside the library, so these tests check that it gives the same
results as ba_fwd (whose workspace the caller allocates) on two calls in a
row, and that it rejects problems too big for the fixed scratch before
running anything. This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import block_sparse_attention_kunlun_b200 as ba
from block_sparse_attention_kunlun_b200.workloads import CONFIGS, make_inputs
from parity_util import check_abs, check_bf16


def test_rejects_problems_beyond_the_fixed_scratch():
    # 1e7 tokens need ~1.2 MiB of tile table: more than the 1 MiB array.
    p = ba.BAProblem(4, 10_000_000, 8, 128, ba.BA_BF16)
    lib = ba._load()
    st = lib.ba_fwd_noalloc(ctypes.byref(p), 1 << 20, 1 << 20, 1 << 20, 1 << 20, 256, 2, None,
                            1 << 20, 1 << 20, None)
    assert st == ba.BA_ERR_INVALID_ARG


@pytest.mark.gpu
def test_noalloc_forward_matches_ba_fwd_twice():
    w = CONFIGS[5].replace(batch=6)
    inp = make_inputs(w, lengths=[300, 2000, 64, 1500, 777, 90])
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    offs = inp["seq_offsets"].cuda()
    skip = inp["skip"].cuda()
    ref_out, ref_lse = ba.block_attention_fwd(q, k, v, offs, w.block, w.window, skip=skip)
    prob = ba.make_problem(q, offs)
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        st = ba.ba_fwd_noalloc(prob, q, k, v, offs, w.block, w.window, skip, out, lse)
        assert st == ba.BA_OK
        torch.cuda.synchronize()
        check_bf16("out", out.cpu(), ref_out.cpu())
        check_abs("lse", lse.cpu(), ref_lse.cpu(), 2e-3)
