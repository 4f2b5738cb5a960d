"""Pins for the MX quantisation oracle (oracle/mx.py).

Each pin checks the oracle against something other than its own code:
- PyTorch's float8_e4m3fn / float8_e5m2 casts (round to nearest even) over
  the range where they are defined (they do not saturate);
- a brute-force nearest search over every element code, decoded from its
  bit pattern, with ties resolved to the even code;
- the scale's definition: a power of two with the block maximum's binade at
  the element format's top exponent; blocks are independent; values that are
  already MX numbers survive the round trip exactly;
- block attention of MX-representable Q and K equals plain block attention.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import mx

TORCH = {"e4m3": torch.float8_e4m3fn, "e5m2": torch.float8_e5m2}


def decode_all(fmt):
    """Every finite element value, decoded from its 8-bit pattern: (values, code is even)."""
    ebits, mbits, bias = (4, 3, 7) if fmt == "e4m3" else (5, 2, 15)
    vals, even = [], []
    for code in range(256):
        s = code >> 7
        ef = (code >> mbits) & ((1 << ebits) - 1)
        mf = code & ((1 << mbits) - 1)
        if fmt == "e4m3" and ef == 15 and mf == 7:
            continue                           # NaN
        if fmt == "e5m2" and ef == 31:
            continue                           # infinities and NaN
        if ef == 0:
            mag = mf * 2.0 ** (1 - bias - mbits)
        else:
            mag = (1 + mf / 2 ** mbits) * 2.0 ** (ef - bias)
        vals.append(-mag if s else mag)
        even.append(mf % 2 == 0)
    return np.array(vals), np.array(even)


def _samples(rng, fmt, n=4000):
    f = mx.FORMATS[fmt]
    # magnitudes spread over every binade of the format, subnormals included, plus exact ties
    exps = rng.uniform(f["emin"] - f["mbits"] - 2, f["emax"] + 0.9, n)
    x = np.exp2(exps) * rng.choice([-1.0, 1.0], n)
    vals, _ = decode_all(fmt)
    pos = np.unique(np.abs(vals))
    ties = (pos[:-1] + pos[1:]) / 2
    return np.concatenate([x, ties[: n // 4], -ties[: n // 4], [0.0, -0.0]])


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_element_rounding_matches_torch_fp8_cast(fmt):
    rng = np.random.default_rng(800)
    x = _samples(rng, fmt)
    x = x[np.abs(x) <= mx.FORMATS[fmt]["maxnorm"]]
    ref = torch.from_numpy(x).to(TORCH[fmt]).double().numpy()
    np.testing.assert_array_equal(mx.round_element(x, fmt), ref)


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_element_rounding_is_nearest_code_ties_to_even(fmt):
    rng = np.random.default_rng(801)
    vals, even = decode_all(fmt)
    x = _samples(rng, fmt, 1500)
    x = x[np.abs(x) <= mx.FORMATS[fmt]["maxnorm"]]
    got = mx.round_element(x, fmt)
    for xi, gi in zip(x, got):
        d = np.abs(vals - xi)
        best = np.flatnonzero(d == d.min())
        if len(set(vals[best])) > 1:           # a tie between two codes: the even one
            best = [b for b in best if even[b]]
        assert gi == vals[best[0]] or (gi == 0 and vals[best[0]] == 0), (xi, gi, vals[best])


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_saturation_above_the_largest_normal(fmt):
    f = mx.FORMATS[fmt]
    x = np.array([f["maxnorm"] * 1.01, f["maxnorm"] * 1.1, 2.0 ** (f["emax"] + 1) * 0.999])
    np.testing.assert_array_equal(mx.round_element(x, fmt), f["maxnorm"])
    np.testing.assert_array_equal(mx.round_element(-x, fmt), -f["maxnorm"])


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_block_scales(fmt):
    rng = np.random.default_rng(802)
    x = rng.standard_normal((5, 3, 96)) * np.exp2(rng.integers(-20, 20, (5, 3, 1)))
    x[0, 0, :32] = 0.0                          # an all-zero block
    el, sc = mx.quantize(x, fmt)
    assert el.shape == (5, 3, 3, 32) and sc.shape == (5, 3, 3, 1)
    np.testing.assert_array_equal(np.exp2(np.round(np.log2(sc))), sc)        # powers of two
    amax = np.max(np.abs(x.reshape(5, 3, 3, 32)), axis=-1, keepdims=True)
    r = (amax / sc)[amax > 0]
    emax = mx.FORMATS[fmt]["emax"]
    assert np.all((r >= 2.0 ** emax) & (r < 2.0 ** (emax + 1)))
    assert not el[0, 0, 0].any()
    # blocks are independent: changing one block leaves the others' results alone
    y = x.copy()
    y[1, 2, 40] *= 1000.0
    a, b = mx.mx_round(x, fmt), mx.mx_round(y, fmt)
    same = np.ones(x.shape, bool)
    same[1, 2, 32:64] = False
    np.testing.assert_array_equal(a[same], b[same])


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_mx_numbers_round_trip_exactly(fmt):
    rng = np.random.default_rng(803)
    vals, _ = decode_all(fmt)
    top = vals[np.abs(vals) >= 2.0 ** mx.FORMATS[fmt]["emax"]]     # the block maximum sits in the top binade
    el = rng.choice(vals, (4, 64))
    el[:, 0] = rng.choice(top, 4)
    el[:, 32] = rng.choice(top, 4)
    el[:, 1:32] = np.clip(el[:, 1:32], -np.abs(el[:, :1]), np.abs(el[:, :1]))
    el[:, 33:] = np.clip(el[:, 33:], -np.abs(el[:, 32:33]), np.abs(el[:, 32:33]))
    x = el * np.exp2(rng.integers(-30, 30, (4, 1)))
    np.testing.assert_array_equal(mx.mx_round(x, fmt), x)


def test_block_maximum_is_rounded_or_clamped():
    """The scale puts the block maximum in [256, 512) (E4M3). Up to the
    largest normal, 448, it is rounded to nearest, within half a unit in its
    4th significant bit; above 448 the rule clamps it to 448 (up to 12.5%
    low). Both happen for Gaussian blocks."""
    rng = np.random.default_rng(804)
    x = rng.standard_normal((400, 32))
    el, sc = mx.quantize(x, "e4m3")
    y = mx.dequantize(el, sc)
    i = np.argmax(np.abs(x), axis=1)
    rows = np.arange(400)
    scaled = np.abs(x[rows, i]) / sc[rows, 0, 0]
    rel = np.abs(y[rows, i] - x[rows, i]) / np.abs(x[rows, i])
    clamped = scaled > 464.0                       # beyond the midpoint of 448 and the next binade value
    assert clamped.any() and (~clamped).any()
    assert np.all(rel[~clamped] <= 2.0 ** -4 * (1 + 1e-12))
    np.testing.assert_array_equal(np.abs(el[rows, 0, i][clamped]), 448.0)


def test_attention_on_mx_representable_operands_is_plain_attention():
    rng = np.random.default_rng(805)
    offs = np.array([0, 40, 40, 77], dtype=np.int32)
    H, D = 2, 64
    q = mx.mx_round(rng.standard_normal((77, H, D)) * 2.0)
    k = mx.mx_round(rng.standard_normal((77, H, D)))
    v = rng.standard_normal((77, H, D))
    a = mx.fwd(offs, q, k, v, 16, 2)
    b = oracle.fwd(offs, q, k, v, 16, 2)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    # and on arbitrary operands the scores move by no more than the quantisation allows
    q2 = rng.standard_normal((77, H, D))
    out_mx, _ = mx.fwd(offs, q2, k, v, 16, 2)
    out, _ = oracle.fwd(offs, q2, k, v, 16, 2)
    assert 0 < np.max(np.abs(out_mx - out)) < 0.1


def test_mx_backward_on_mx_representable_operands_is_plain_backward():
    rng = np.random.default_rng(806)
    offs = np.array([0, 40, 40, 77], dtype=np.int32)
    H, D = 2, 64
    q = mx.mx_round(rng.standard_normal((77, H, D)) * 2.0)
    k = mx.mx_round(rng.standard_normal((77, H, D)))
    v, do = rng.standard_normal((77, H, D)), rng.standard_normal((77, H, D))
    for x, y in zip(mx.bwd(offs, q, k, v, do, 16, 2), oracle.bwd(offs, q, k, v, do, 16, 2)):
        np.testing.assert_array_equal(x, y)


def test_mx_backward_is_straight_through_autograd():
    """The backward against PyTorch autograd of masked attention whose q and k
    pass through the MX round trip in the forward and straight through it in
    the backward (x + (round(x) - x).detach()), fp64, per example."""
    rng = np.random.default_rng(807)
    block, window, H, D = 8, 2, 2, 64
    offs = np.array([0, 23, 23, 60], dtype=np.int32)
    T = int(offs[-1])
    q, k = rng.standard_normal((T, H, D)) * 1.5, rng.standard_normal((T, H, D))
    v, do = rng.standard_normal((T, H, D)), rng.standard_normal((T, H, D))
    dq, dk, dv = mx.bwd(offs, q, k, v, do, block, window)
    plain = oracle.bwd(offs, q, k, v, do, block, window)
    assert np.max(np.abs(dq - plain[0])) > 1e-6  # the rounding is not skipped
    for e in range(len(offs) - 1):
        s0, s1 = int(offs[e]), int(offs[e + 1])
        L = s1 - s0
        if L == 0:
            continue
        i = torch.arange(L)[:, None]
        j = torch.arange(L)[None, :]
        mask = (j <= i) & (j // block >= i // block - (window - 1))
        tq, tk, tv = (torch.tensor(x[s0:s1].transpose(1, 0, 2), dtype=torch.float64, requires_grad=True)
                      for x in (q, k, v))
        rq = torch.tensor(mx.mx_round(q[s0:s1]).transpose(1, 0, 2))
        rk = torch.tensor(mx.mx_round(k[s0:s1]).transpose(1, 0, 2))
        o = torch.nn.functional.scaled_dot_product_attention(tq + (rq - tq).detach(), tk + (rk - tk).detach(), tv,
                                                             attn_mask=mask)
        o.backward(torch.tensor(do[s0:s1].transpose(1, 0, 2)))
        t = lambda x: x.detach().numpy().transpose(1, 0, 2)
        for name, got, ref in (("dq", dq, tq.grad), ("dk", dk, tk.grad), ("dv", dv, tv.grad)):
            np.testing.assert_allclose(got[s0:s1], t(ref), rtol=0, atol=1e-11, err_msg=f"{name} example {e}")
