"""The FMA-pipe 2^x that the bf16 softmax uses for part of its exponentials
(to take load off the special-function unit), through ba_selftest_exp2,
against 2^x evaluated in fp64 on the host.

Stated bound (include/ba.h): relative error below 1e-4 for x in [-125, 8],
the range the kernels feed it (scores minus a running maximum that may lag
the true one by up to 8 in log2 units); x below -125 gives at most 2^-125.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_kunlun_b200 as ba

pytestmark = pytest.mark.gpu


def gpu_exp2(x: np.ndarray) -> np.ndarray:
    xd = torch.from_numpy(x.astype(np.float32)).cuda()
    yd = torch.empty_like(xd)
    assert ba.ba_selftest_exp2(xd, yd) == ba.BA_OK
    torch.cuda.synchronize()
    return yd.cpu().numpy().astype(np.float64)


def test_fma_exp2_relative_error_on_a_dense_grid():
    grid = np.linspace(-125.0, 8.0, 1 << 22, dtype=np.float64).astype(np.float32)
    # both sides of every rounding split at n + 1/2, and the integers themselves
    n = np.arange(-125, 9, dtype=np.float64)
    half = np.concatenate([n + 0.5, n]).astype(np.float32)
    edges = np.concatenate([np.nextafter(half, np.float32(-np.inf)), half, np.nextafter(half, np.float32(np.inf))])
    x = np.concatenate([grid, edges[(edges >= -125) & (edges <= 8)]])
    y = gpu_exp2(x)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 1e-4, f"max relative error {rel.max():.3e} at x = {x[np.argmax(rel)]}"


def test_fma_exp2_below_the_range_stays_tiny():
    x = np.array([-125.5, -126, -130, -149, -200, -1e30, -np.inf], dtype=np.float32)
    y = gpu_exp2(x)
    assert np.all(y >= 0) and np.all(y <= 2.0 ** -125 * (1 + 1e-4))
