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
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

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
