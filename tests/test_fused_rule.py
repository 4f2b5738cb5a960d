"""The fused-backward dispatch rule against the mask rule, on the CPU.

The bf16 backward runs as one fused pass exactly when every 128-row query
tile of an example sees keys of its own 128-row key tile only (each
example's tiles start at its first row). The library decides this from
(block, window) alone, and the choice shows on the host in the backward's
workspace size: the fused pass adds one staged region of k rows. Here the
mask rule (query i sees key j iff j <= i and j // block >= i // block -
(window - 1), local indices) is evaluated by brute force for every query of
a ragged multi-tile example, and the library's choice must match it for
every block up to 300 and windows 1 to 4. bench.py's own copy of the rule
(which labels the kernels it times) is checked the same way.
"""
import numpy as np

import block_sparse_attention_kunlun_b200 as ba
from block_sparse_attention_kunlun_b200.workloads import CONFIGS
import bench

TILE = 128
L = 8 * TILE + 37  # several full tiles and a ragged tail


def own_tile_only(block, window):
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    seen = (j <= i) & (j // block >= i // block - (window - 1))
    return bool(np.all(~seen | (j // TILE == i // TILE)))


def prob():
    return ba.BAProblem(3, 1000, 2, 128, ba.BA_BF16)


def test_library_runs_the_fused_pass_exactly_when_tiles_see_only_themselves():
    p = prob()
    base = ba.ba_bwd_workspace_size(p, 256, 2)  # a mask that crosses tiles: the two-pass backward
    staged_k = (3 * TILE * 2 * 128 * 2 + 255) // 256 * 256
    fused_seen = []
    for window in (1, 2, 3, 4):
        for block in range(1, 301):
            extra = ba.ba_bwd_workspace_size(p, block, window) - base
            assert extra in (0, staged_k), (block, window, extra)
            fused = extra == staged_k
            assert fused == own_tile_only(block, window), (block, window)
            if fused:
                fused_seen.append(block)
    # the blocks that qualify: window 1 and the divisors of 128
    assert fused_seen == [1, 2, 4, 8, 16, 32, 64, 128]


def test_bench_labels_the_fused_pass_by_the_same_rule():
    for window in (1, 2, 3):
        for block in range(1, 301):
            w = CONFIGS[3].replace(block=block, window=window)
            assert bench.fused_backward(w) == own_tile_only(block, window), (block, window)
            assert not bench.fused_backward(w, rope=True) and not bench.fused_backward(w, gdpa="gelu")
    # float32 has no fused backward
    assert not bench.fused_backward(CONFIGS[1].replace(block=64, window=1))
