"""CPU oracle for generalized dot-product attention (TEST INFRASTRUCTURE ONLY).

Only the tests may import this module; the library never does.

What it computes. "Meta Scales GEM Ads Model Across Platforms and Thousands of
GPUs" (opening section) lists Generalized Dot-Product Attention among GEM's
recommendation-specific kernels. "GEM (Meta)", section "Custom kernels", says
it serves GEM's self-attention, cross-attention and pooled multi-head
attention, with the softmax replaced by an activation such as GELU or SiLU,
and that it is fastest on short keys/values. "Scaling Meta's Generative Ads
Model (GEM) for Ads Recommendations", section "Kunlun Architecture Details",
adds that per-example feed-forward networks were reformulated into it. The
pages give no formula. The plainest reading, used here:

  s_ij   = (q_i . k_j) / sqrt(D)               (the attention's scaled score)
  out_i  = sum_{j visible to i} act(s_ij) v_j  (no normalisation: the
                                               activation takes the softmax's
                                               place and nothing else changes)
  act    = GELU (x Phi(x), Phi the standard normal CDF, exact erf form) or
           SiLU (x sigmoid(x))

Backward (exact gradient of out for upstream dO):
  dA_ij = dO_i . v_j,   dS_ij = act'(s_ij) dA_ij     (visible pairs only)
  dq_i  = (1/sqrt(D)) sum_j dS_ij k_j
  dk_j  = (1/sqrt(D)) sum_i dS_ij q_i
  dv_j  = sum_i act(s_ij) dO_i

Visibility: self-attention over a jagged batch uses the block rule of the rest
of this project (query i sees key j iff j <= i and
floor(j/block) >= floor(i/block) - (window-1), local indices). Cross-attention
(and pooled attention, which is cross-attention whose queries are a set of
seeds) gives every query of example b every key of example b's own key/value
set; the two sets are jagged separately.

Everything is fp64, dense per (example, head), with the visibility mask
written out for every pair. Pins: tests/test_oracle_gdpa.py.
"""
from __future__ import annotations

import numpy as np
from scipy.special import erf

ACTIVATIONS = ("gelu", "silu")


def act(x, kind):
    """The activation that replaces the softmax."""
    x = np.asarray(x, dtype=np.float64)
    if kind == "gelu":
        return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))
    if kind == "silu":
        with np.errstate(over="ignore"):
            return x / (1.0 + np.exp(-x))
    raise ValueError(f"unknown activation {kind!r}")


def act_grad(x, kind):
    """Derivative of act: GELU' = Phi(x) + x phi(x); SiLU' = sigma(x) (1 + x (1 - sigma(x)))."""
    x = np.asarray(x, dtype=np.float64)
    if kind == "gelu":
        return 0.5 * (1.0 + erf(x / np.sqrt(2.0))) + x * np.exp(-0.5 * x * x) / np.sqrt(2.0 * np.pi)
    if kind == "silu":
        with np.errstate(over="ignore"):
            sg = 1.0 / (1.0 + np.exp(-x))
        return sg * (1.0 + x * (1.0 - sg))
    raise ValueError(f"unknown activation {kind!r}")


def block_mask(L, block, window):
    """[L, L] boolean: query i (row) sees key j (column) under the block rule."""
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    return (j <= i) & (j // block >= i // block - (window - 1))


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _check(offsets, *ts):
    offs = np.asarray(offsets, dtype=np.int64)
    if offs.ndim != 1 or offs[0] != 0 or np.any(np.diff(offs) < 0) or offs[-1] != ts[0].shape[0]:
        raise ValueError("offsets must start at 0, be non-decreasing and end at the row count")
    return offs


def _pair_fwd(qe, ke, ve, mask, kind):
    """One (example, head): qe [Lq, D], ke/ve [Lk, D], mask [Lq, Lk] or None."""
    s = (qe @ ke.T) / np.sqrt(qe.shape[1])
    a = act(s, kind)
    if mask is not None:
        a = np.where(mask, a, 0.0)
    return a @ ve


def _pair_bwd(qe, ke, ve, de, mask, kind):
    scale = 1.0 / np.sqrt(qe.shape[1])
    s = (qe @ ke.T) * scale
    a = act(s, kind)
    ds = act_grad(s, kind) * (de @ ve.T)
    if mask is not None:
        a = np.where(mask, a, 0.0)
        ds = np.where(mask, ds, 0.0)
    return scale * (ds @ ke), scale * (ds.T @ qe), a.T @ de


def fwd(seq_offsets, q, k, v, block, window, activation):
    """Self-attention GDPA over a jagged batch: q, k, v [T, H, D] -> out [T, H, D]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    offs = _check(seq_offsets, q, k, v)
    out = np.zeros_like(q)
    for e in range(len(offs) - 1):
        s0, s1 = int(offs[e]), int(offs[e + 1])
        if s1 == s0:
            continue
        m = block_mask(s1 - s0, block, window)
        for h in range(q.shape[1]):
            out[s0:s1, h] = _pair_fwd(q[s0:s1, h], k[s0:s1, h], v[s0:s1, h], m, activation)
    return out


def bwd(seq_offsets, q, k, v, dout, block, window, activation):
    """Gradients of fwd for upstream dout. Returns (dq, dk, dv)."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    offs = _check(seq_offsets, q, k, v)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(q), np.zeros_like(q)
    for e in range(len(offs) - 1):
        s0, s1 = int(offs[e]), int(offs[e + 1])
        if s1 == s0:
            continue
        m = block_mask(s1 - s0, block, window)
        for h in range(q.shape[1]):
            sl = slice(s0, s1)
            dq[sl, h], dk[sl, h], dv[sl, h] = _pair_bwd(q[sl, h], k[sl, h], v[sl, h], dout[sl, h], m, activation)
    return dq, dk, dv


def cross_fwd(q_offsets, kv_offsets, q, k, v, activation):
    """Cross-attention GDPA: example b's queries (rows q_offsets[b]..) see
    every key of its own key/value rows (kv_offsets[b]..). q [Tq, H, D],
    k, v [Tk, H, D] -> out [Tq, H, D]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    qo = _check(q_offsets, q)
    ko = _check(kv_offsets, k, v)
    if len(qo) != len(ko):
        raise ValueError("q_offsets and kv_offsets must describe the same number of examples")
    out = np.zeros_like(q)
    for e in range(len(qo) - 1):
        a0, a1, b0, b1 = int(qo[e]), int(qo[e + 1]), int(ko[e]), int(ko[e + 1])
        if a1 == a0 or b1 == b0:
            continue   # no queries, or no keys: the sum is empty
        for h in range(q.shape[1]):
            out[a0:a1, h] = _pair_fwd(q[a0:a1, h], k[b0:b1, h], v[b0:b1, h], None, activation)
    return out


def cross_bwd(q_offsets, kv_offsets, q, k, v, dout, activation):
    """Gradients of cross_fwd. Returns (dq, dk, dv)."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    qo = _check(q_offsets, q)
    ko = _check(kv_offsets, k, v)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for e in range(len(qo) - 1):
        a0, a1, b0, b1 = int(qo[e]), int(qo[e + 1]), int(ko[e]), int(ko[e + 1])
        if a1 == a0 or b1 == b0:
            continue
        for h in range(q.shape[1]):
            dq[a0:a1, h], dk[b0:b1, h], dv[b0:b1, h] = _pair_bwd(
                q[a0:a1, h], k[b0:b1, h], v[b0:b1, h], dout[a0:a1, h], None, activation)
    return dq, dk, dv
