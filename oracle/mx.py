"""MX block quantisation (MXFP8) and block attention on MXFP8 operands
(TEST INFRASTRUCTURE ONLY; only the tests may import this module).

What it computes. "Meta Scales GEM Ads Model Across Platforms and Thousands
of GPUs" (opening section) says GEM trains attention and feed-forward layers
in MXFP8 precision. The pages define neither the format nor which operands
it covers. The format is the public OCP Microscaling (MX) one, restated
here from its definition:

  - a block of 32 consecutive elements along the contraction dimension
    shares one scale X = 2^e, an 8-bit exponent (E8M0, e in [-127, 127]);
  - each element is an FP8 number: E4M3 (3 mantissa bits, exponents -6..8,
    largest normal 448, no infinities) or E5M2 (2 mantissa bits, exponents
    -14..15, largest normal 57344);
  - quantising a block: e = floor(log2(max |v|)) - emax, where emax is the
    element format's largest exponent (8 for E4M3, 15 for E5M2); each v / X
    is rounded to the nearest element value, ties to even, and magnitudes
    above the largest normal are clamped to it.

Reading for attention (the plainest one the sentence supports): the
operands of the score product Q K^T are MXFP8, blocked along head_dim, the
contraction of that product. The softmax and P V are unchanged, so the
result is block attention of the dequantised Q and K. The backward, which
the same sentence puts in MXFP8 too, recomputes the scores from the same
MXFP8 Q and K and passes the gradient through the quantisation unchanged
(its derivative taken as the identity, the usual reading for training
through a rounding step): dq and dk are the gradients with respect to the
dequantised operands. Everything else is the fp64 oracle of
oracle/oracle.c. Pins: tests/test_oracle_mx.py.
"""
from __future__ import annotations

import numpy as np

import oracle

BLOCK = 32

# element formats: mantissa bits, smallest normal exponent, largest exponent, largest normal value
FORMATS = {
    "e4m3": dict(mbits=3, emin=-6, emax=8, maxnorm=448.0),
    "e5m2": dict(mbits=2, emin=-14, emax=15, maxnorm=57344.0),
}


def round_element(x, fmt):
    """Round x (already divided by its block scale) to the element format:
    nearest value, ties to even, subnormals below 2^emin, magnitudes above
    the largest normal clamped to it."""
    f = FORMATS[fmt]
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    # the value's binade, floored at the smallest normal exponent (subnormals share its quantum)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, f["emin"])
    quantum = np.exp2(e - f["mbits"])
    r = np.round(a / quantum) * quantum          # numpy rounds halves to even
    r = np.minimum(r, f["maxnorm"])
    return np.copysign(r, x)


def quantize(x, fmt="e4m3"):
    """MX quantisation of x along its last axis (a multiple of 32 long).
    Returns (elements [..., n/32, 32] as element-format values, scales
    [..., n/32, 1] as powers of two)."""
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    if n % BLOCK:
        raise ValueError("the blocked axis must be a multiple of 32 long")
    b = x.reshape(x.shape[:-1] + (n // BLOCK, BLOCK))
    amax = np.max(np.abs(b), axis=-1, keepdims=True)
    e = np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - FORMATS[fmt]["emax"]
    scale = np.exp2(np.clip(e, -127, 127))
    return round_element(b / scale, fmt), scale


def dequantize(elements, scale):
    """Inverse view of quantize: element values times their block's scale,
    with the blocked axis flattened back."""
    v = elements * scale
    return v.reshape(v.shape[:-2] + (v.shape[-2] * v.shape[-1],))


def mx_round(x, fmt="e4m3"):
    """x after an MX quantise / dequantise round trip along its last axis."""
    return dequantize(*quantize(x, fmt))


def fwd(seq_offsets, q, k, v, block, window, fmt="e4m3", skip=None, nthreads=None):
    """Block attention with Q and K as MXFP8 operands (blocks of 32 along
    head_dim). Returns (out, lse) like oracle.fwd."""
    return oracle.fwd(seq_offsets, mx_round(q, fmt), mx_round(k, fmt), v, block, window, skip=skip,
                      nthreads=nthreads)


def bwd(seq_offsets, q, k, v, dout, block, window, fmt="e4m3", skip=None, nthreads=None):
    """Backward of fwd: the gradients of block attention of the dequantised
    Q and K, taken with respect to those dequantised operands (the rounding
    passed through unchanged). Returns (dq, dk, dv) like oracle.bwd."""
    return oracle.bwd(seq_offsets, mx_round(q, fmt), mx_round(k, fmt), v, dout, block, window, skip=skip,
                      nthreads=nthreads)
