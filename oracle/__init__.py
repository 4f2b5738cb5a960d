"""CPU oracle for block attention (TEST INFRASTRUCTURE ONLY).

Plain fp64 dense-mask block attention, forward and backward, written in C
(``oracle.c``) and loaded here through ctypes. Only the tests, the smoke check
and the benchmark's CPU-baseline leg may import this package; the library
never does, and it has no CPU fallback.

The rule it implements (stated on no page; fixed for the whole project): a
query at local index i of an example sees key j iff j <= i and
floor(j/block) >= floor(i/block) - (window-1). See ``oracle.c`` for the full
definition and for the passages of the pages it follows ("Meta Scales GEM Ads
Model Across Platforms and Thousands of GPUs", section "Kunlun changes how GEM
scales"; "GEM (Meta)", sections "Custom kernels" and "Training
infrastructure").

Every function takes numpy arrays: q, k, v, dout as float64 [T, H, D]
(C-contiguous), seq_offsets as int32 [batch + 1], skip as uint8 [batch] or
None. Pins: tests/test_oracle.py.

Rotary position embedding (``rope_*``; "GEM (Meta)", section "Custom
kernels": the production block-attention kernel fuses the backward pass of
the rotary position embedding; the pages say nothing more about it). The
reading used here and in the library is RoFormer's rotation applied to q and
k (not v) before the scores: the adjacent pair (x[2k], x[2k+1]) of a row at
position p is turned by the angle whose cosine and sine the caller's tables
hold at [p, k]; p is the row's index within its example, the origin the
blocks use. The gradient with respect to the unrotated q (k) is the
transposed rotation of the gradient with respect to the rotated q (k).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (portable x86-64 code)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
             "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i32 = ctypes.c_int32
        lib.oracle_fwd.argtypes = [i32, P, i32, i32, i32, i32, P, P, P, P, P, P, i32]
        lib.oracle_fwd.restype = ctypes.c_int
        lib.oracle_bwd.argtypes = [i32, P, i32, i32, i32, i32, P, P, P, P, P, P, P, P, i32]
        lib.oracle_bwd.restype = ctypes.c_int
        lib.oracle_rows.argtypes = [i32, i32, i32, i32, i32, i32, P, P, P, P, i32, P,
                                    P, P, P, P, P, i32]
        lib.oracle_rows.restype = ctypes.c_int
        _lib = lib
    return _lib


def default_threads() -> int:
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)


def _f64(a):
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _prep(seq_offsets, q, k, v, skip):
    offs = np.ascontiguousarray(seq_offsets, dtype=np.int32)
    q, k, v = _f64(q), _f64(k), _f64(v)
    if q.ndim != 3 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share shape [T, H, D]")
    batch = offs.shape[0] - 1
    if batch < 0 or offs[0] != 0 or offs[-1] != q.shape[0] or np.any(np.diff(offs) < 0):
        raise ValueError("seq_offsets must start at 0, be non-decreasing and end at T")
    if skip is not None:
        skip = np.ascontiguousarray(skip, dtype=np.uint8)
        if skip.shape != (batch,):
            raise ValueError("skip must have one flag per example")
    return offs, batch, q, k, v, skip


def fwd(seq_offsets, q, k, v, block, window, skip=None, nthreads=None):
    """Forward pass. Returns (out [T, H, D] float64, lse [H, T] float64)."""
    offs, batch, q, k, v, skip = _prep(seq_offsets, q, k, v, skip)
    T, H, D = q.shape
    out = np.empty_like(q)
    lse = np.empty((H, T), dtype=np.float64)
    rc = _load().oracle_fwd(batch, _ptr(offs), H, D, int(block), int(window), _ptr(skip),
                            _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                            int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle_fwd failed ({rc})")
    return out, lse


def bwd(seq_offsets, q, k, v, dout, block, window, skip=None, nthreads=None):
    """Backward pass for upstream gradient dout. Returns (dq, dk, dv)."""
    offs, batch, q, k, v, skip = _prep(seq_offsets, q, k, v, skip)
    dout = _f64(dout)
    if dout.shape != q.shape:
        raise ValueError("dout must have the shape of q")
    T, H, D = q.shape
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    rc = _load().oracle_bwd(batch, _ptr(offs), H, D, int(block), int(window), _ptr(skip),
                            _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                            int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle_bwd failed ({rc})")
    return dq, dk, dv


def rows(q_e, k_e, v_e, head, rows_idx, block, window, dout_e=None,
         want=("out", "lse"), nthreads=None):
    """Selected local rows of one (example, head).

    q_e, k_e, v_e (and dout_e for gradients) are the example's own rows,
    [L, H, D]. ``want`` names any of out, lse, dq, dk, dv; returns a dict of
    float64 arrays ([n, D], or [n] for lse) in the order of ``rows_idx``.
    """
    q_e, k_e, v_e = _f64(q_e), _f64(k_e), _f64(v_e)
    L, H, D = q_e.shape
    r = np.ascontiguousarray(rows_idx, dtype=np.int32)
    n = r.shape[0]
    res = {}
    for name in want:
        res[name] = np.empty((n,) if name == "lse" else (n, D), dtype=np.float64)
    if any(w in res for w in ("dq", "dk", "dv")):
        if dout_e is None:
            raise ValueError("gradients need dout_e")
        dout_e = _f64(dout_e)
    rc = _load().oracle_rows(L, H, D, int(block), int(window), int(head),
                             _ptr(q_e), _ptr(k_e), _ptr(v_e), _ptr(dout_e), n, _ptr(r),
                             _ptr(res.get("out")), _ptr(res.get("lse")), _ptr(res.get("dq")),
                             _ptr(res.get("dk")), _ptr(res.get("dv")),
                             int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle_rows failed ({rc})")
    return res


# ------------------------------------------------------------ rotary ---

def positions(seq_offsets):
    """Local position of every row: its index within its own example."""
    offs = np.asarray(seq_offsets, dtype=np.int64)
    lens = np.diff(offs)
    return np.arange(int(offs[-1]), dtype=np.int64) - np.repeat(offs[:-1], lens)


def _rotate_at(x, pos, cos, sin, transpose):
    """Rotate the adjacent pairs of rows x[n, ..., D] sitting at positions pos[n]:
    y[2k] = x[2k] c - x[2k+1] s, y[2k+1] = x[2k] s + x[2k+1] c with c, s the
    tables' entries at [pos, k], in fp64. transpose=True applies the
    transposed 2 x 2 map instead (c, s) -> (c, -s), which takes a gradient
    with respect to y to the gradient with respect to x; it is also the
    inverse when the tables hold exact cosines and sines."""
    x = _f64(x)
    cos = np.asarray(cos, dtype=np.float64)
    sin = np.asarray(sin, dtype=np.float64)
    D = x.shape[-1]
    if D % 2 or cos.ndim != 2 or cos.shape[1] != D // 2 or sin.shape != cos.shape:
        raise ValueError("rotary tables must be [rows, head_dim / 2] with an even head_dim")
    pos = np.asarray(pos, dtype=np.int64)
    if pos.size and (pos.min() < 0 or pos.max() >= cos.shape[0]):
        raise ValueError("rotary tables are shorter than an example")
    shape = (pos.shape[0],) + (1,) * (x.ndim - 2) + (D // 2,)
    c = cos[pos].reshape(shape)
    s = sin[pos].reshape(shape)
    if transpose:
        s = -s
    x0, x1 = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = x0 * c - x1 * s
    y[..., 1::2] = x0 * s + x1 * c
    return y


def rope_rotate(x, seq_offsets, cos, sin, transpose=False):
    """Rotary embedding of every row of x [T, H, D] at its local position, in
    fp64 (transpose=True: the transposed rotation)."""
    return _rotate_at(x, positions(seq_offsets), cos, sin, transpose)


def round_bf16(x):
    """Round fp64 values to the nearest bfloat16 value, ties to the even
    significand, straight from the definition: bfloat16 keeps 8 significant
    bits and float32's exponent range, so with x = m 2^e (0.5 <= |m| < 1) the
    result is rint(m 2^8) 2^(e - 8); numpy's rint rounds half to even and
    m 2^8 is exact in fp64. Only finite values inside bfloat16's normal range
    are used here (|x| in [2^-126, 2^128) or 0)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


def _rotated_operand(x, seq_offsets, cos, sin, operand_dtype):
    """The rotated q or k as the attention's products take it. None: the
    exact fp64 rotation. torch.bfloat16: that exact rotation rounded to the
    nearest bfloat16 value (ties to even), the operand type of a library
    whose tensor-core products take the input dtype."""
    y = rope_rotate(x, seq_offsets, cos, sin)
    if operand_dtype is None:
        return y
    if operand_dtype != torch.bfloat16:
        raise ValueError("operand_dtype must be None or torch.bfloat16")
    return round_bf16(y)


def rope_fwd(seq_offsets, q, k, v, cos, sin, block, window, skip=None, operand_dtype=None, nthreads=None):
    """Block attention of the rotated q and k. operand_dtype=torch.bfloat16
    rounds the exact rotated q and k to bfloat16 first, as a library that
    feeds them to tensor-core products in the input dtype holds them."""
    qr = _rotated_operand(q, seq_offsets, cos, sin, operand_dtype)
    kr = _rotated_operand(k, seq_offsets, cos, sin, operand_dtype)
    return fwd(seq_offsets, qr, kr, v, block, window, skip=skip, nthreads=nthreads)


def rope_bwd(seq_offsets, q, k, v, dout, cos, sin, block, window, skip=None, operand_dtype=None,
             nthreads=None):
    """Gradients of rope_fwd: dv as for plain attention, dq and dk the
    transposed rotations of the gradients with respect to the rotated q and
    k (the rounding of operand_dtype counts as the identity)."""
    qr = _rotated_operand(q, seq_offsets, cos, sin, operand_dtype)
    kr = _rotated_operand(k, seq_offsets, cos, sin, operand_dtype)
    dqr, dkr, dv = bwd(seq_offsets, qr, kr, v, dout, block, window, skip=skip, nthreads=nthreads)
    return (rope_rotate(dqr, seq_offsets, cos, sin, transpose=True),
            rope_rotate(dkr, seq_offsets, cos, sin, transpose=True), dv)


def rope_rows(q_e, k_e, v_e, cos, sin, head, rows_idx, block, window, dout_e=None,
              want=("out", "lse"), operand_dtype=None, nthreads=None):
    """``rows`` for the rotated attention of one example (rows [L, H, D])."""
    L = _f64(q_e).shape[0]
    offs = np.array([0, L], dtype=np.int32)
    qr = _rotated_operand(q_e, offs, cos, sin, operand_dtype)
    kr = _rotated_operand(k_e, offs, cos, sin, operand_dtype)
    res = rows(qr, kr, v_e, head, rows_idx, block, window, dout_e=dout_e, want=want, nthreads=nthreads)
    pos = np.asarray(rows_idx, dtype=np.int64)
    for name in ("dq", "dk"):
        if name in res:
            res[name] = _rotate_at(res[name], pos, cos, sin, transpose=True)
    return res
