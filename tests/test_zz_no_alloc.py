"""The forward entry point that allocates nothing (ba_fwd_noalloc).

It exists for callers that cannot call cudaMalloc, such as a framework that
owns all device memory through its own pool and hands kernels only their
inputs and outputs. Its scratch is a fixed 1 MiB array inside the library,
so these tests check that it gives exactly the results of ba_fwd (whose
workspace the caller allocates; both run the same kernels on the same
inputs, so the bits must agree) on two calls in a row, and that problems too
big for the fixed scratch are rejected. This file is collected last on
purpose.
"""
import ctypes

import pytest
import torch

import block_sparse_attention_kunlun_b200 as ba
from block_sparse_attention_kunlun_b200.workloads import CONFIGS, make_inputs

SCRATCH = 1 << 20


def _largest_single_example_tokens():
    """The longest single example (in whole 128-row tiles) whose forward
    workspace fits the fixed scratch, found from ba_fwd_workspace_size."""
    lo, hi = 128, 1 << 24
    while hi - lo > 128:
        mid = (lo + hi) // 2 // 128 * 128
        p = ba.BAProblem(1, mid, 1, 64, ba.BA_BF16)
        if ba.ba_fwd_workspace_size(p, 64, 1) <= SCRATCH:
            lo = mid
        else:
            hi = mid
    return lo


def test_size_limit_of_the_fixed_scratch():
    t = _largest_single_example_tokens()
    assert 5_000_000 < t < 6_000_000  # about 5.5 million tokens for one example
    over = ba.BAProblem(1, t + 128, 1, 64, ba.BA_BF16)
    assert ba.ba_fwd_workspace_size(over, 64, 1) > SCRATCH
    # a problem over the limit is rejected; every pointer is NULL, so even a call
    # that got past the size check would be turned away before any launch
    big = ba.BAProblem(4, 10_000_000, 8, 128, ba.BA_BF16)
    assert ba.ba_fwd_workspace_size(big, 256, 2) > SCRATCH
    lib = ba._load()
    for p in (over, big):
        st = lib.ba_fwd_noalloc(ctypes.byref(p), None, None, None, None, 256, 2, None, None, None, None)
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
        assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)


@pytest.mark.gpu
def test_noalloc_accepts_the_largest_problem_that_fits():
    """One example at the size limit runs and matches ba_fwd bit for bit; one
    tile more is rejected before anything runs."""
    t = _largest_single_example_tokens()
    gen = torch.Generator(device="cuda")
    gen.manual_seed(7)
    q, k, v = (torch.randn((t, 1, 64), generator=gen, device="cuda").to(torch.bfloat16) for _ in range(3))
    offs = torch.tensor([0, t], dtype=torch.int32, device="cuda")
    prob = ba.make_problem(q, offs)
    out = torch.empty_like(q)
    lse = torch.empty((1, t), dtype=torch.float32, device="cuda")
    assert ba.ba_fwd_noalloc(prob, q, k, v, offs, 64, 1, None, out, lse) == ba.BA_OK
    ref_out, ref_lse = ba.block_attention_fwd(q, k, v, offs, 64, 1)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
    over = ba.BAProblem(1, t + 128, 1, 64, ba.BA_BF16)
    # NULL pointers: these tensors are one tile too short for `over`
    assert ba.ba_fwd_noalloc(over, None, None, None, None, 64, 1, None, None, None) == ba.BA_ERR_INVALID_ARG
