"""A second, literal block-attention forward used only to pin the oracle.

Written independently of oracle/oracle.c: for every query it lists the keys
the rule allows (no matrix, no mask array, no max shift) and forms the
softmax-weighted sum with exactly rounded sums (math.fsum). Only for tiny
inputs: pure Python loops.
"""
import math


def visible_keys(i, block, window):
    first_block = max(0, i // block - (window - 1))
    return list(range(first_block * block, i + 1))


def fwd(offsets, q, k, v, block, window):
    """q, k, v: numpy float64 [T, H, D]. Returns (out [T,H,D] list, lse [H][T])."""
    T, H, D = q.shape
    out = [[[0.0] * D for _ in range(H)] for _ in range(T)]
    lse = [[0.0] * T for _ in range(H)]
    scale = 1.0 / math.sqrt(D)
    for e in range(len(offsets) - 1):
        s0, s1 = int(offsets[e]), int(offsets[e + 1])
        for h in range(H):
            for i in range(s1 - s0):
                keys = visible_keys(i, block, window)
                w = []
                for j in keys:
                    dot = math.fsum(float(q[s0 + i, h, d]) * float(k[s0 + j, h, d]) for d in range(D))
                    w.append(math.exp(dot * scale))
                z = math.fsum(w)
                for d in range(D):
                    out[s0 + i][h][d] = math.fsum(wj * float(v[s0 + j, h, d]) for wj, j in zip(w, keys)) / z
                lse[h][s0 + i] = math.log(z)
    return out, lse
