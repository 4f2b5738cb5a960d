"""Pins for the CPU oracle (oracle/): checks against facts fixed outside it.

Each test pins the oracle to something other than itself: hand-derived
values (tests/golden/), a second literal implementation (tests/brute.py),
library routines in special cases that reduce to them (PyTorch's causal
scaled-dot-product attention and autograd, in fp64), calculus (finite
differences, softmax sum identities) and structural facts (examples are
independent; one-block and window-1 rules).
"""
import math
import os

import numpy as np
import pytest
import torch

import brute
import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def rand_case(rng, lengths, H, D, scale=1.0):
    offs = np.zeros(len(lengths) + 1, dtype=np.int32)
    offs[1:] = np.cumsum(lengths)
    T = int(offs[-1])
    q = rng.standard_normal((T, H, D)) * scale
    k = rng.standard_normal((T, H, D)) * scale
    v = rng.standard_normal((T, H, D))
    do = rng.standard_normal((T, H, D))
    return offs, q, k, v, do


# ---------------------------------------------------------------- golden ---

def load_masks():
    tables, cur = [], None
    with open(os.path.join(GOLDEN, "masks.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("mask"):
                _, L, b, w = line.split()
                cur = (int(L), int(b), int(w), [])
                tables.append(cur)
            else:
                cur[3].append([int(c) for c in line])
    return tables


@pytest.mark.parametrize("table", load_masks(), ids=lambda t: f"L{t[0]}_b{t[1]}_w{t[2]}")
def test_mask_tables_by_hand(table):
    """q = k = 0 makes every visible key equally likely; with one-hot values
    the output row is 1/count at exactly the visible keys."""
    L, block, window, rows = table
    mask = np.array(rows, dtype=np.float64)
    assert mask.shape == (L, L)
    offs = np.array([0, L], dtype=np.int32)
    q = np.zeros((L, 1, 1))
    k = np.zeros((L, 1, 1))
    v = np.eye(L).reshape(L, 1, L)
    q = np.zeros((L, 1, L))
    k = np.zeros((L, 1, L))
    out, lse = oracle.fwd(offs, q, k, v, block, window)
    count = mask.sum(1)
    np.testing.assert_array_equal(out[:, 0, :] > 0, mask > 0)
    np.testing.assert_allclose(out[:, 0, :], mask / count[:, None], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[0], np.log(count), rtol=0, atol=1e-15)


def load_worked():
    vals = {}
    with open(os.path.join(GOLDEN, "worked_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            w, name, *xs = line.split()
            vals[(int(w), name)] = np.array([eval(x, {"math": math}) for x in xs])
    return vals


@pytest.mark.parametrize("window", [1, 2])
def test_worked_example_by_hand(window):
    g = load_worked()
    offs = np.array([0, 3], dtype=np.int32)
    q = np.ones((3, 1, 1))
    k = np.array([0.0, math.log(3), math.log(2)]).reshape(3, 1, 1)
    v = np.array([4.0, 8.0, -1.0]).reshape(3, 1, 1)
    do = np.ones((3, 1, 1))
    out, lse = oracle.fwd(offs, q, k, v, 2, window)
    dq, dk, dv = oracle.bwd(offs, q, k, v, do, 2, window)
    for name, got in [("out", out[:, 0, 0]), ("lse", lse[0]), ("dq", dq[:, 0, 0]),
                      ("dk", dk[:, 0, 0]), ("dv", dv[:, 0, 0])]:
        np.testing.assert_allclose(got, g[(window, name)], rtol=0, atol=1e-14, err_msg=name)


# ----------------------------------------------------------- brute force ---

@pytest.mark.parametrize("seed", range(6))
def test_matches_literal_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    block = [1, 2, 3, 5, 8, 4][seed]
    window = [1, 2, 3, 2, 1, 3][seed]
    D = [1, 4, 3, 4, 1, 2][seed]
    H = 1 + seed % 2
    lengths = [int(x) for x in rng.integers(0, 40, size=3)] + [1]
    offs, q, k, v, _ = rand_case(rng, lengths, H, D)
    out, lse = oracle.fwd(offs, q, k, v, block, window)
    bout, blse = brute.fwd(offs, q, k, v, block, window)
    np.testing.assert_allclose(out, np.array(bout).reshape(out.shape), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, np.array(blse).reshape(lse.shape), rtol=0, atol=1e-12)


# ------------------------------------------------- library special cases ---

def sdpa_causal(q, k, v, dout):
    """PyTorch causal attention (fp64) for one example [L, H, D]; returns out and grads."""
    tq, tk, tv = (torch.tensor(x.transpose(1, 0, 2), dtype=torch.float64, requires_grad=True)
                  for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    o.backward(torch.tensor(dout.transpose(1, 0, 2)))
    t = lambda x: x.detach().numpy().transpose(1, 0, 2)
    return t(o), t(tq.grad), t(tk.grad), t(tv.grad)


@pytest.mark.parametrize("block,window,lengths", [
    (16, 4, [64, 37, 1, 50]),      # window * block = 64 >= every length
    (64, 1, [64, 10, 33]),          # one block covers everything
    (7, 10, [70, 69, 3]),
])
def test_full_causal_when_window_covers_sequence(block, window, lengths):
    rng = np.random.default_rng(7)
    offs, q, k, v, do = rand_case(rng, lengths, 3, 8)
    out, _ = oracle.fwd(offs, q, k, v, block, window)
    dq, dk, dv = oracle.bwd(offs, q, k, v, do, block, window)
    for e in range(len(lengths)):
        s, t = offs[e], offs[e + 1]
        if t == s:
            continue
        ro, rdq, rdk, rdv = sdpa_causal(q[s:t], k[s:t], v[s:t], do[s:t])
        np.testing.assert_allclose(out[s:t], ro, rtol=0, atol=1e-12)
        np.testing.assert_allclose(dq[s:t], rdq, rtol=0, atol=1e-12)
        np.testing.assert_allclose(dk[s:t], rdk, rtol=0, atol=1e-12)
        np.testing.assert_allclose(dv[s:t], rdv, rtol=0, atol=1e-12)


def test_window1_is_causal_attention_per_block():
    """window = 1: the pages' independent blocks, each a causal attention of its own."""
    rng = np.random.default_rng(8)
    block = 8
    lengths = [29, 8, 17]
    offs, q, k, v, do = rand_case(rng, lengths, 2, 4)
    out, _ = oracle.fwd(offs, q, k, v, block, 1)
    dq, dk, dv = oracle.bwd(offs, q, k, v, do, block, 1)
    for e in range(len(lengths)):
        for c0 in range(offs[e], offs[e + 1], block):
            c1 = min(c0 + block, offs[e + 1])
            ro, rdq, rdk, rdv = sdpa_causal(q[c0:c1], k[c0:c1], v[c0:c1], do[c0:c1])
            np.testing.assert_allclose(out[c0:c1], ro, rtol=0, atol=1e-12)
            np.testing.assert_allclose(dq[c0:c1], rdq, rtol=0, atol=1e-12)
            np.testing.assert_allclose(dk[c0:c1], rdk, rtol=0, atol=1e-12)
            np.testing.assert_allclose(dv[c0:c1], rdv, rtol=0, atol=1e-12)


def test_short_example_needs_one_block():
    """An example no longer than one block gives the same result for every window."""
    rng = np.random.default_rng(9)
    offs, q, k, v, do = rand_case(rng, [16, 5, 1], 2, 4)
    ref = oracle.fwd(offs, q, k, v, 16, 1)
    refg = oracle.bwd(offs, q, k, v, do, 16, 1)
    for window in (2, 3, 7):
        out, lse = oracle.fwd(offs, q, k, v, 16, window)
        np.testing.assert_array_equal(out, ref[0])
        np.testing.assert_array_equal(lse, ref[1])
        for a, b in zip(oracle.bwd(offs, q, k, v, do, 16, window), refg):
            np.testing.assert_array_equal(a, b)


# ------------------------------------------------------------ closed form ---

def test_first_row_of_each_block_has_one_key():
    """With window 1 the first query of every block sees only itself: o = v
    exactly and lse = its own scaled score."""
    rng = np.random.default_rng(10)
    block = 5
    offs, q, k, v, _ = rand_case(rng, [23, 5, 11], 2, 6)
    out, lse = oracle.fwd(offs, q, k, v, block, 1)
    for e in range(3):
        for i in range(0, offs[e + 1] - offs[e], block):
            r = offs[e] + i
            np.testing.assert_array_equal(out[r], v[r])
            for h in range(2):
                assert lse[h, r] == pytest.approx(q[r, h] @ k[r, h] / math.sqrt(6), abs=1e-14)


def test_gradient_sum_identities():
    """Softmax rows sum to one, so sum_j dv_j = sum_i dO_i; and each row of ds
    sums to zero, so sum_j dk_j = 0 (per example and head)."""
    rng = np.random.default_rng(11)
    offs, q, k, v, do = rand_case(rng, [40, 13, 64], 2, 5)
    dq, dk, dv = oracle.bwd(offs, q, k, v, do, 8, 2)
    for e in range(3):
        s, t = offs[e], offs[e + 1]
        np.testing.assert_allclose(dv[s:t].sum(0), do[s:t].sum(0), rtol=0, atol=1e-12)
        np.testing.assert_allclose(dk[s:t].sum(0), 0.0, rtol=0, atol=1e-12)


def test_finite_differences():
    rng = np.random.default_rng(12)
    block, window = 3, 2
    offs, q, k, v, do = rand_case(rng, [9, 4], 1, 3)
    dq, dk, dv = oracle.bwd(offs, q, k, v, do, block, window)
    eps = 1e-6

    def f(q_, k_, v_):
        return float(np.sum(oracle.fwd(offs, q_, k_, v_, block, window)[0] * do))

    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            num[idx] = (f(*args_p) - f(*args_m)) / (2 * eps)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8, err_msg=name)


# ------------------------------------------------------------- structure ---

def test_jagged_batch_equals_separate_runs_and_permutes():
    rng = np.random.default_rng(13)
    lengths = [31, 0, 17, 45]
    offs, q, k, v, do = rand_case(rng, lengths, 2, 4)
    out, lse = oracle.fwd(offs, q, k, v, 8, 2)
    dq, dk, dv = oracle.bwd(offs, q, k, v, do, 8, 2)
    for e in range(len(lengths)):
        s, t = offs[e], offs[e + 1]
        one = np.array([0, t - s], dtype=np.int32)
        o1, l1 = oracle.fwd(one, q[s:t], k[s:t], v[s:t], 8, 2)
        np.testing.assert_array_equal(out[s:t], o1)
        np.testing.assert_array_equal(lse[:, s:t], l1)
        g1 = oracle.bwd(one, q[s:t], k[s:t], v[s:t], do[s:t], 8, 2)
        for a, b in zip((dq, dk, dv), g1):
            np.testing.assert_array_equal(a[s:t], b)
    perm = [3, 0, 2, 1]
    idx = np.concatenate([np.arange(offs[e], offs[e + 1]) for e in perm])
    poffs = np.zeros(5, dtype=np.int32)
    poffs[1:] = np.cumsum([lengths[e] for e in perm])
    po, pl = oracle.fwd(poffs, q[idx], k[idx], v[idx], 8, 2)
    np.testing.assert_array_equal(po, out[idx])
    np.testing.assert_array_equal(pl, lse[:, idx])


def test_skip_passes_values_through():
    rng = np.random.default_rng(14)
    offs, q, k, v, do = rand_case(rng, [20, 9, 33], 2, 4)
    skip = np.array([1, 0, 1], dtype=np.uint8)
    out, lse = oracle.fwd(offs, q, k, v, 4, 2, skip=skip)
    dq, dk, dv = oracle.bwd(offs, q, k, v, do, 4, 2, skip=skip)
    ref_o, ref_l = oracle.fwd(offs, q, k, v, 4, 2)
    ref_g = oracle.bwd(offs, q, k, v, do, 4, 2)
    for e in range(3):
        s, t = offs[e], offs[e + 1]
        if skip[e]:
            np.testing.assert_array_equal(out[s:t], v[s:t])
            np.testing.assert_array_equal(lse[:, s:t], 0.0)
            np.testing.assert_array_equal(dq[s:t], 0.0)
            np.testing.assert_array_equal(dk[s:t], 0.0)
            np.testing.assert_array_equal(dv[s:t], do[s:t])
        else:
            np.testing.assert_array_equal(out[s:t], ref_o[s:t])
            np.testing.assert_array_equal(lse[:, s:t], ref_l[:, s:t])
            for a, b in zip((dq, dk, dv), ref_g):
                np.testing.assert_array_equal(a[s:t], b[s:t])


def test_sampled_rows_match_full_computation():
    rng = np.random.default_rng(15)
    L = 57
    offs, q, k, v, do = rand_case(rng, [L], 3, 4)
    out, lse = oracle.fwd(offs, q, k, v, 6, 3)
    dq, dk, dv = oracle.bwd(offs, q, k, v, do, 6, 3)
    rows = [0, 5, 6, 17, 56, 30]
    for h in range(3):
        r = oracle.rows(q, k, v, h, rows, 6, 3, dout_e=do, want=("out", "lse", "dq", "dk", "dv"))
        np.testing.assert_allclose(r["out"], out[rows, h], rtol=0, atol=1e-13)
        np.testing.assert_allclose(r["lse"], lse[h, rows], rtol=0, atol=1e-13)
        np.testing.assert_allclose(r["dq"], dq[rows, h], rtol=0, atol=1e-13)
        np.testing.assert_allclose(r["dk"], dk[rows, h], rtol=0, atol=1e-13)
        np.testing.assert_allclose(r["dv"], dv[rows, h], rtol=0, atol=1e-13)


def test_thread_count_does_not_change_bits():
    rng = np.random.default_rng(16)
    offs, q, k, v, do = rand_case(rng, [30, 44, 12, 50], 3, 4)
    a = oracle.fwd(offs, q, k, v, 8, 2, nthreads=1) + oracle.bwd(offs, q, k, v, do, 8, 2, nthreads=1)
    b = oracle.fwd(offs, q, k, v, 8, 2, nthreads=5) + oracle.bwd(offs, q, k, v, do, 8, 2, nthreads=5)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


# --------------------------------------------- sliding-window attention ---
# Token-granular sliding window ("GEM (Meta)", "Custom kernels": the
# predecessor of block attention): query i sees keys i - w < j <= i. The
# library runs it as the block rule with block = 1; these pins check that
# reading against the window rule written out directly.

def _swa_brute_fwd(offsets, q, k, v, w):
    T, H, D = q.shape
    out = np.zeros((T, H, D))
    lse = np.zeros((H, T))
    scale = 1.0 / math.sqrt(D)
    for e in range(len(offsets) - 1):
        s0, s1 = int(offsets[e]), int(offsets[e + 1])
        for h in range(H):
            for i in range(s1 - s0):
                keys = [j for j in range(s1 - s0) if i - w < j <= i]
                wts = [math.exp(math.fsum(q[s0 + i, h, d] * k[s0 + j, h, d] for d in range(D)) * scale)
                       for j in keys]
                z = math.fsum(wts)
                for d in range(D):
                    out[s0 + i, h, d] = math.fsum(a * v[s0 + j, h, d] for a, j in zip(wts, keys)) / z
                lse[h, s0 + i] = math.log(z)
    return out, lse


@pytest.mark.parametrize("w", [1, 2, 5, 17])
def test_sliding_window_is_block_rule_with_block_1(w):
    rng = np.random.default_rng(300 + w)
    offs, q, k, v, _ = rand_case(rng, [23, 0, 9, 31], 2, 3)
    out, lse = oracle.fwd(offs, q, k, v, 1, w)
    bout, blse = _swa_brute_fwd(offs, q, k, v, w)
    np.testing.assert_allclose(out, bout, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, blse, rtol=0, atol=1e-12)


def test_sliding_window_gradients_match_masked_sdpa():
    """Backward against PyTorch attention with an explicit band mask (fp64)."""
    rng = np.random.default_rng(41)
    L, H, D, w = 40, 2, 8, 7
    offs, q, k, v, do = rand_case(rng, [L], H, D)
    dq, dk, dv = oracle.bwd(offs, q, k, v, do, 1, w)
    i = torch.arange(L)[:, None]
    j = torch.arange(L)[None, :]
    band = (j <= i) & (j > i - w)
    tq, tk, tv = (torch.tensor(x.transpose(1, 0, 2), dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=band)
    o.backward(torch.tensor(do.transpose(1, 0, 2)))
    for name, got, ref in (("dq", dq, tq.grad), ("dk", dk, tk.grad), ("dv", dv, tv.grad)):
        np.testing.assert_allclose(got, ref.numpy().transpose(1, 0, 2), rtol=0, atol=1e-11, err_msg=name)


# ------------------------------------------------- rotary embedding ---
# Rotary position embedding on q and k ("GEM (Meta)", "Custom kernels": the
# block-attention kernel fuses the backward pass of the rotary embedding).
# RoFormer writes the rotation as a complex multiplication: the pair
# (x[2k], x[2k+1]) read as x[2k] + i x[2k+1] is multiplied by exp(i p theta_k).
# These pins check the oracle's real-arithmetic form against that, against
# autograd through it, and against the relative-position property it exists
# for.

def _exact_tables(rows, D, base=10000.0):
    ang = np.arange(rows, dtype=np.float64)[:, None] * base ** (-2.0 * np.arange(D // 2) / D)[None, :]
    return np.cos(ang), np.sin(ang), ang


def _complex_rotate(x, pos, ang):
    z = x[..., 0::2] + 1j * x[..., 1::2]
    z = z * np.exp(1j * ang[pos])[:, None, :]
    y = np.empty_like(x)
    y[..., 0::2] = z.real
    y[..., 1::2] = z.imag
    return y


def test_rope_rotation_is_complex_multiplication():
    rng = np.random.default_rng(500)
    offs, q, _, _, _ = rand_case(rng, [17, 0, 40, 5], 3, 8)
    cos, sin, ang = _exact_tables(64, 8)
    pos = np.concatenate([np.arange(17), np.arange(40), np.arange(5)])
    np.testing.assert_allclose(oracle.rope_rotate(q, offs, cos, sin), _complex_rotate(q, pos, ang),
                               rtol=0, atol=1e-13)
    # the transpose turns by the opposite angle: multiplication by the conjugate
    np.testing.assert_allclose(oracle.rope_rotate(q, offs, cos, sin, transpose=True),
                               _complex_rotate(q, pos, -ang), rtol=0, atol=1e-13)


def test_rope_transpose_undoes_rotation_and_keeps_pair_norms():
    rng = np.random.default_rng(501)
    offs, q, _, _, _ = rand_case(rng, [33, 12], 2, 16)
    cos, sin, _ = _exact_tables(40, 16)
    y = oracle.rope_rotate(q, offs, cos, sin)
    np.testing.assert_allclose(oracle.rope_rotate(y, offs, cos, sin, transpose=True), q, rtol=0, atol=1e-13)
    np.testing.assert_allclose(np.hypot(y[..., 0::2], y[..., 1::2]), np.hypot(q[..., 0::2], q[..., 1::2]),
                               rtol=1e-13, atol=0)


def test_rope_attention_depends_on_relative_position_only():
    """RoFormer's property: rotating every position by a further constant
    angle leaves q . k, hence out and lse, unchanged."""
    rng = np.random.default_rng(502)
    offs, q, k, v, _ = rand_case(rng, [45, 30], 2, 8, scale=2.0)
    cos, sin, ang = _exact_tables(100, 8)
    out0, lse0 = oracle.rope_fwd(offs, q, k, v, cos, sin, 8, 3)
    out1, lse1 = oracle.rope_fwd(offs, q, k, v, np.cos(ang[37:]), np.sin(ang[37:]), 8, 3)
    np.testing.assert_allclose(out1, out0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse1, lse0, rtol=0, atol=1e-12)
    # ... while a table that is not a rotation by p * theta does change them
    out2, _ = oracle.rope_fwd(offs, q, k, v, cos[::-1].copy(), sin[::-1].copy(), 8, 3)
    assert np.max(np.abs(out2 - out0)) > 1e-3


def test_rope_gradients_match_autograd_of_complex_form():
    """Backward against PyTorch autograd through the complex-number rotation
    followed by masked attention (fp64), per example, jagged batch."""
    rng = np.random.default_rng(503)
    block, window, H, D = 4, 2, 2, 8
    offs, q, k, v, do = rand_case(rng, [13, 0, 29], H, D, scale=1.5)
    cos, sin, ang = _exact_tables(32, D)
    dq, dk, dv = oracle.rope_bwd(offs, q, k, v, do, cos, sin, block, window)
    out, _ = oracle.rope_fwd(offs, q, k, v, cos, sin, block, window)
    for e in range(len(offs) - 1):
        s0, s1 = int(offs[e]), int(offs[e + 1])
        L = s1 - s0
        if L == 0:
            continue
        i = torch.arange(L)[:, None]
        j = torch.arange(L)[None, :]
        mask = (j <= i) & (j // block >= i // block - (window - 1))
        rot = torch.polar(torch.ones(L, D // 2, dtype=torch.float64),
                          torch.tensor(ang[:L]))[None, :, :]                      # [1, L, D/2]
        tq, tk, tv = (torch.tensor(x[s0:s1].transpose(1, 0, 2), dtype=torch.float64, requires_grad=True)
                      for x in (q, k, v))
        as_c = lambda t: torch.view_as_complex(t.reshape(H, L, D // 2, 2))
        as_r = lambda z: torch.view_as_real(z).reshape(H, L, D)
        o = torch.nn.functional.scaled_dot_product_attention(as_r(as_c(tq) * rot), as_r(as_c(tk) * rot), tv,
                                                             attn_mask=mask)
        o.backward(torch.tensor(do[s0:s1].transpose(1, 0, 2)))
        t = lambda x: x.detach().numpy().transpose(1, 0, 2)
        np.testing.assert_allclose(out[s0:s1], t(o), rtol=0, atol=1e-12)
        for name, got, ref in (("dq", dq, tq.grad), ("dk", dk, tk.grad), ("dv", dv, tv.grad)):
            np.testing.assert_allclose(got[s0:s1], t(ref), rtol=0, atol=1e-11, err_msg=f"{name} example {e}")


def test_rope_identity_tables_give_plain_attention():
    rng = np.random.default_rng(504)
    offs, q, k, v, do = rand_case(rng, [20, 7], 2, 4)
    one, zero = np.ones((20, 2)), np.zeros((20, 2))
    for a, b in zip(oracle.rope_fwd(offs, q, k, v, one, zero, 4, 2), oracle.fwd(offs, q, k, v, 4, 2)):
        np.testing.assert_array_equal(a, b)
    for a, b in zip(oracle.rope_bwd(offs, q, k, v, do, one, zero, 4, 2), oracle.bwd(offs, q, k, v, do, 4, 2)):
        np.testing.assert_array_equal(a, b)


def test_rope_positions_restart_in_every_example():
    """A jagged batch equals each example run alone (positions are local);
    dq and dk, unlike out, depend on the absolute position, so they would
    differ if positions ran over the whole batch."""
    rng = np.random.default_rng(505)
    offs, q, k, v, do = rand_case(rng, [21, 34], 2, 8)
    cos, sin, _ = _exact_tables(64, 8)
    dq, dk, dv = oracle.rope_bwd(offs, q, k, v, do, cos, sin, 8, 2)
    s = slice(21, 55)
    one = np.array([0, 34], dtype=np.int32)
    dq1, dk1, dv1 = oracle.rope_bwd(one, q[s], k[s], v[s], do[s], cos, sin, 8, 2)
    np.testing.assert_allclose(dq[s], dq1, rtol=0, atol=1e-13)
    np.testing.assert_allclose(dk[s], dk1, rtol=0, atol=1e-13)
    np.testing.assert_allclose(dv[s], dv1, rtol=0, atol=1e-13)
    glob = np.arange(55)[s]   # rows numbered over the batch instead
    dq_glob = oracle._rotate_at(oracle.rope_rotate(dq1, one, cos, sin), glob, cos, sin, transpose=True)
    assert np.max(np.abs(dq_glob - dq[s])) > 1e-3


def test_rope_rows_match_full_computation():
    rng = np.random.default_rng(506)
    offs, q, k, v, do = rand_case(rng, [70], 2, 8)
    cos, sin, _ = _exact_tables(80, 8)
    out, lse = oracle.rope_fwd(offs, q, k, v, cos, sin, 16, 2)
    dq, dk, dv = oracle.rope_bwd(offs, q, k, v, do, cos, sin, 16, 2)
    idx = np.array([0, 5, 16, 31, 69])
    r = oracle.rope_rows(q, k, v, cos, sin, 1, idx, 16, 2, dout_e=do, want=("out", "lse", "dq", "dk", "dv"))
    for name, full in (("out", out), ("dq", dq), ("dk", dk), ("dv", dv)):
        np.testing.assert_allclose(r[name], full[idx, 1], rtol=0, atol=1e-13, err_msg=name)
    np.testing.assert_allclose(r["lse"], lse[1, idx], rtol=0, atol=1e-13)


def test_rope_tables_shorter_than_an_example_are_rejected():
    offs, q, k, v, _ = rand_case(np.random.default_rng(507), [10, 12], 1, 4)
    cos, sin, _ = _exact_tables(11, 4)
    with pytest.raises(ValueError):
        oracle.rope_fwd(offs, q, k, v, cos, sin, 4, 1)


def _bf16_neighbours(x):
    """The two bfloat16 values around each fp64 x (x > 0), found by walking
    float32 bit patterns whose low 16 bits are zero."""
    f = np.float32(x)
    bits = np.array([f]).view(np.uint32)[0] & np.uint32(0xFFFF0000)
    lo = np.array([bits], dtype=np.uint32).view(np.float32)[0].astype(np.float64)
    if lo > x:
        bits -= np.uint32(0x10000)
        lo = np.array([bits], dtype=np.uint32).view(np.float32)[0].astype(np.float64)
    hi_bits = bits + np.uint32(0x10000)
    hi = np.array([hi_bits], dtype=np.uint32).view(np.float32)[0].astype(np.float64)
    return lo, hi, int(bits >> 16) & 1


def test_round_bf16_is_nearest_with_ties_to_even():
    """round_bf16 (the rounding of the rotated operands) against a brute-force
    search of the two neighbouring bfloat16 values, exact midpoints (which
    go to the even significand), values a hair off a midpoint (where
    rounding through float32 first would land on the midpoint and go the
    wrong way), and torch's float32 -> bfloat16 cast on float32 inputs."""
    rng = np.random.default_rng(497)
    xs = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-6, 6, 2000),
                         rng.uniform(0.5, 8.0, 200)])
    got = oracle.round_bf16(xs)
    for x, g in zip(xs, got):
        a = abs(x)
        lo, hi, lo_odd = _bf16_neighbours(a)
        want = lo if (a - lo < hi - a or (a - lo == hi - a and not lo_odd)) else hi
        assert g == np.copysign(want, x), (x, g, want)
    for a in (1.0, 3.0, 0.0078125, 1000.0):
        lo, hi, lo_odd = _bf16_neighbours(a * (1 + 2.0 ** -20))
        mid = (lo + hi) / 2
        assert oracle.round_bf16(mid) == (hi if lo_odd else lo)
        assert oracle.round_bf16(-mid) == -(hi if lo_odd else lo)
        # just above the midpoint rounds up, even where float32 would first round onto the midpoint
        above = mid * (1 + 2.0 ** -40)
        assert np.float32(above) == np.float32(mid)
        assert oracle.round_bf16(above) == hi
    f32 = rng.standard_normal(5000).astype(np.float32)
    ref = torch.from_numpy(f32).to(torch.bfloat16).double().numpy()
    assert np.array_equal(oracle.round_bf16(f32.astype(np.float64)), ref)
    assert oracle.round_bf16(np.array([0.0]))[0] == 0.0


def test_rotated_bf16_operands_are_the_exact_rotation_rounded():
    rng = np.random.default_rng(508)
    offs, q, _, _, _ = rand_case(rng, [50, 30], 2, 16, scale=3.0)
    q = torch.from_numpy(q).to(torch.bfloat16).double().numpy()
    cos, sin, _ = _exact_tables(64, 16)
    exact = oracle.rope_rotate(q, offs, cos, sin)
    a = oracle._rotated_operand(q, offs, cos, sin, torch.bfloat16)
    assert np.array_equal(a, oracle.round_bf16(exact))
    assert np.array_equal(oracle._rotated_operand(q, offs, cos, sin, None), exact)
    # each rounded value is within half a bfloat16 step of the exact one
    step = 2.0 ** (np.floor(np.log2(np.abs(exact))) - 7)
    assert np.all(np.abs(a - exact) <= step / 2)
