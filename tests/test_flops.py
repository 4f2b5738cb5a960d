"""Pins for the benchmark's work accounting (host logic, no GPU)."""
import numpy as np

from block_sparse_attention_kunlun_b200 import flops as F
from test_oracle import load_masks


def test_pair_counts_match_hand_written_masks():
    for L, block, window, rows in load_masks():
        assert F.visible_pairs([L], block, window) == int(np.array(rows).sum())


def test_pair_counts_brute_force_and_skip():
    rng = np.random.default_rng(3)
    for _ in range(20):
        lens = [int(x) for x in rng.integers(0, 300, size=4)]
        block, window = int(rng.integers(1, 70)), int(rng.integers(1, 5))
        skip = rng.integers(0, 2, size=4)
        brute = 0
        for e, L in enumerate(lens):
            if skip[e]:
                continue
            for i in range(L):
                for j in range(i + 1):
                    if j // block >= i // block - (window - 1):
                        brute += 1
        assert F.visible_pairs(lens, block, window, skip) == brute
        assert F.live_tokens(lens, skip) == sum(L for L, s in zip(lens, skip) if not s)


def test_full_attention_limit_and_flop_split():
    # a window covering everything gives L (L + 1) / 2 pairs
    assert F.visible_pairs([1000], 64, 10**6) == 1000 * 1001 // 2
    f = F.step_flops(10, 2, 64)
    assert f["fwd"] == 4 * 64 * 20 and f["bwd"] == 10 * 64 * 20 and f["step"] == 14 * 64 * 20
