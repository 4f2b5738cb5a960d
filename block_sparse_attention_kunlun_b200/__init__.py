"""Block attention for NVIDIA B200 (sm_100a).

Python binding over the C ABI in ``include/ba.h`` (``libba.so`` in this
package directory, built by ``build.py``). The functions named like the C
entry points (``ba_fwd``, ``ba_bwd``, ...) marshal torch tensors into
pointers and call the library; every step of the computation runs in the
library's CUDA kernels. There is no CPU path: if the library is missing or
the device is not an sm_100 GPU, the calls raise.

Tensors: q, k, v, out, dout, dq, dk, dv are contiguous CUDA tensors of shape
``[total_tokens, heads, head_dim]`` (bfloat16 or float32); lse is float32
``[heads, total_tokens]``; seq_offsets is int32 ``[batch + 1]`` on the
device; skip is uint8 ``[batch]`` on the device or None.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "BAError", "ba_fwd", "ba_fwd_noalloc", "ba_bwd", "ba_fwd_workspace_size", "ba_bwd_workspace_size",
    "ba_swa_fwd", "ba_swa_bwd", "ba_swa_fwd_workspace_size", "ba_swa_bwd_workspace_size",
    "ba_rope_fwd", "ba_rope_bwd", "ba_rope_fwd_workspace_size", "ba_rope_bwd_workspace_size",
    "ba_device_status", "ba_selftest_wait_timeout", "ba_selftest_exp2", "ba_selftest_activation", "ba_set_profile_events", "ba_status_string", "ba_version",
    "block_attention_fwd", "block_attention_bwd", "sliding_window_attention_fwd", "sliding_window_attention_bwd",
    "rope_block_attention_fwd", "rope_block_attention_bwd",
    "ba_gdpa_workspace_size", "ba_gdpa_fwd", "ba_gdpa_bwd", "gdpa_fwd", "gdpa_bwd",
    "ba_gdpa_cross_workspace_size", "ba_gdpa_cross_fwd", "ba_gdpa_cross_bwd", "gdpa_cross_fwd", "gdpa_cross_bwd",
    "ba_mx_quantize", "ba_mx_fwd_workspace_size", "ba_mx_fwd", "mx_quantize", "mx_block_attention_fwd",
    "ba_mx_bwd_workspace_size", "ba_mx_bwd", "mx_block_attention_bwd",
    "library_path",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libba.so")

BA_OK, BA_ERR_INVALID_ARG, BA_ERR_UNSUPPORTED, BA_ERR_CUDA, BA_ERR_TIMEOUT = range(5)
BA_F32, BA_BF16 = 0, 1
BA_ACT_GELU, BA_ACT_SILU = 1, 2
_ACTS = {"gelu": BA_ACT_GELU, "silu": BA_ACT_SILU}
_DTYPES = {torch.float32: BA_F32, torch.bfloat16: BA_BF16}


class BAProblem(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("total_tokens", ctypes.c_int32),
                ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("dtype", ctypes.c_int)]


class BARope(ctypes.Structure):
    _fields_ = [("cos", ctypes.c_void_p), ("sin", ctypes.c_void_p), ("rows", ctypes.c_int32),
                ("q_rot", ctypes.c_void_p), ("k_rot", ctypes.c_void_p)]


class BAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {ba_status_string(status)} ({status})")


_lib = None


def library_path() -> str:
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with "
                          "`python -m block_sparse_attention_kunlun_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    P, i32 = ctypes.c_void_p, ctypes.c_int32
    prob = ctypes.POINTER(BAProblem)
    lib.ba_fwd_workspace_size.argtypes = [prob, i32, i32]
    lib.ba_fwd_workspace_size.restype = ctypes.c_size_t
    lib.ba_bwd_workspace_size.argtypes = [prob, i32, i32]
    lib.ba_bwd_workspace_size.restype = ctypes.c_size_t
    lib.ba_fwd.argtypes = [prob, P, P, P, P, i32, i32, P, P, P, P, ctypes.c_size_t, P]
    lib.ba_fwd.restype = ctypes.c_int
    lib.ba_bwd.argtypes = [prob, P, P, P, P, P, P, P, i32, i32, P, P, P, P, P, ctypes.c_size_t, P]
    lib.ba_bwd.restype = ctypes.c_int
    lib.ba_device_status.argtypes = [P, P]
    lib.ba_device_status.restype = ctypes.c_int
    lib.ba_status_string.argtypes = [ctypes.c_int]
    lib.ba_status_string.restype = ctypes.c_char_p
    lib.ba_fwd_noalloc.argtypes = [prob, P, P, P, P, i32, i32, P, P, P, P]
    lib.ba_fwd_noalloc.restype = ctypes.c_int
    lib.ba_set_profile_events.argtypes = [i32, P, P]
    lib.ba_set_profile_events.restype = ctypes.c_int
    lib.ba_version.argtypes = []
    lib.ba_version.restype = ctypes.c_int32
    lib.ba_selftest_wait_timeout.argtypes = [P, ctypes.c_size_t, i32, P]
    lib.ba_selftest_wait_timeout.restype = ctypes.c_int
    lib.ba_selftest_exp2.argtypes = [P, P, ctypes.c_int64, P]
    lib.ba_selftest_exp2.restype = ctypes.c_int
    lib.ba_selftest_activation.argtypes = [ctypes.c_int, P, P, P, ctypes.c_int64, P]
    lib.ba_selftest_activation.restype = ctypes.c_int
    lib.ba_swa_fwd_workspace_size.argtypes = [prob, i32]
    lib.ba_swa_fwd_workspace_size.restype = ctypes.c_size_t
    lib.ba_swa_bwd_workspace_size.argtypes = [prob, i32]
    lib.ba_swa_bwd_workspace_size.restype = ctypes.c_size_t
    lib.ba_swa_fwd.argtypes = [prob, P, P, P, P, i32, P, P, P, P, ctypes.c_size_t, P]
    lib.ba_swa_fwd.restype = ctypes.c_int
    lib.ba_swa_bwd.argtypes = [prob, P, P, P, P, P, P, P, i32, P, P, P, P, P, ctypes.c_size_t, P]
    lib.ba_swa_bwd.restype = ctypes.c_int
    lib.ba_gdpa_workspace_size.argtypes = [prob, i32, i32]
    lib.ba_gdpa_workspace_size.restype = ctypes.c_size_t
    lib.ba_gdpa_fwd.argtypes = [prob, ctypes.c_int, P, P, P, P, i32, i32, P, P, ctypes.c_size_t, P]
    lib.ba_gdpa_fwd.restype = ctypes.c_int
    lib.ba_gdpa_bwd.argtypes = [prob, ctypes.c_int, P, P, P, P, P, i32, i32, P, P, P, P, ctypes.c_size_t, P]
    lib.ba_gdpa_bwd.restype = ctypes.c_int
    lib.ba_gdpa_cross_workspace_size.argtypes = [prob, i32]
    lib.ba_gdpa_cross_workspace_size.restype = ctypes.c_size_t
    lib.ba_gdpa_cross_fwd.argtypes = [prob, i32, ctypes.c_int, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    lib.ba_gdpa_cross_fwd.restype = ctypes.c_int
    lib.ba_gdpa_cross_bwd.argtypes = [prob, i32, ctypes.c_int, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    lib.ba_gdpa_cross_bwd.restype = ctypes.c_int
    lib.ba_mx_quantize.argtypes = [P, ctypes.c_int64, i32, i32, P, P, P]
    lib.ba_mx_quantize.restype = ctypes.c_int
    lib.ba_mx_fwd_workspace_size.argtypes = [prob, i32, i32]
    lib.ba_mx_fwd_workspace_size.restype = ctypes.c_size_t
    lib.ba_mx_fwd.argtypes = [prob, P, P, P, P, i32, i32, P, P, P, P, ctypes.c_size_t, P]
    lib.ba_mx_fwd.restype = ctypes.c_int
    lib.ba_mx_bwd_workspace_size.argtypes = [prob, i32, i32]
    lib.ba_mx_bwd_workspace_size.restype = ctypes.c_size_t
    lib.ba_mx_bwd.argtypes = [prob, P, P, P, P, P, P, P, i32, i32, P, P, P, P, P, ctypes.c_size_t, P]
    lib.ba_mx_bwd.restype = ctypes.c_int
    rope = ctypes.POINTER(BARope)
    lib.ba_rope_fwd_workspace_size.argtypes = [prob, i32, i32]
    lib.ba_rope_fwd_workspace_size.restype = ctypes.c_size_t
    lib.ba_rope_bwd_workspace_size.argtypes = [prob, i32, i32]
    lib.ba_rope_bwd_workspace_size.restype = ctypes.c_size_t
    lib.ba_rope_fwd.argtypes = [prob, rope, P, P, P, P, i32, i32, P, P, P, P, ctypes.c_size_t, P]
    lib.ba_rope_fwd.restype = ctypes.c_int
    lib.ba_rope_bwd.argtypes = [prob, rope, P, P, P, P, P, P, P, i32, i32, P, P, P, P, P, ctypes.c_size_t, P]
    lib.ba_rope_bwd.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_problem(q: torch.Tensor, seq_offsets: torch.Tensor) -> BAProblem:
    if q.dim() != 3:
        raise ValueError("q must be [total_tokens, heads, head_dim]")
    if q.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {q.dtype}")
    T, H, D = q.shape
    return BAProblem(int(seq_offsets.numel()) - 1, T, H, D, _DTYPES[q.dtype])


def ba_status_string(status: int) -> str:
    return _load().ba_status_string(int(status)).decode()


def ba_version() -> int:
    return int(_load().ba_version())


def ba_fwd_workspace_size(problem: BAProblem, block: int, window: int) -> int:
    return int(_load().ba_fwd_workspace_size(ctypes.byref(problem), int(block), int(window)))


def ba_bwd_workspace_size(problem: BAProblem, block: int, window: int) -> int:
    return int(_load().ba_bwd_workspace_size(ctypes.byref(problem), int(block), int(window)))


def ba_fwd(problem, q, k, v, seq_offsets, block, window, skip, out, lse, workspace,
           workspace_bytes=None, stream=None) -> int:
    """Direct call of the C entry point; returns its status code."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return int(_load().ba_fwd(ctypes.byref(problem), _ptr(q), _ptr(k), _ptr(v), _ptr(seq_offsets),
                              int(block), int(window), _ptr(skip), _ptr(out), _ptr(lse),
                              _ptr(workspace), int(workspace_bytes), _stream(stream)))


def ba_fwd_noalloc(problem, q, k, v, seq_offsets, block, window, skip, out, lse, stream=None) -> int:
    """Direct call of the no-allocation forward (scratch inside the library)."""
    return int(_load().ba_fwd_noalloc(ctypes.byref(problem), _ptr(q), _ptr(k), _ptr(v), _ptr(seq_offsets),
                                      int(block), int(window), _ptr(skip), _ptr(out), _ptr(lse),
                                      _stream(stream)))


def ba_bwd(problem, q, k, v, out, lse, dout, seq_offsets, block, window, skip, dq, dk, dv,
           workspace, workspace_bytes=None, stream=None) -> int:
    """Direct call of the C entry point; returns its status code."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return int(_load().ba_bwd(ctypes.byref(problem), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                              _ptr(dout), _ptr(seq_offsets), int(block), int(window), _ptr(skip),
                              _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), int(workspace_bytes),
                              _stream(stream)))


def ba_swa_fwd_workspace_size(problem: BAProblem, window_tokens: int) -> int:
    return int(_load().ba_swa_fwd_workspace_size(ctypes.byref(problem), int(window_tokens)))


def ba_swa_bwd_workspace_size(problem: BAProblem, window_tokens: int) -> int:
    return int(_load().ba_swa_bwd_workspace_size(ctypes.byref(problem), int(window_tokens)))


def ba_swa_fwd(problem, q, k, v, seq_offsets, window_tokens, skip, out, lse, workspace,
               workspace_bytes=None, stream=None) -> int:
    """Direct call of the sliding-window forward; returns its status code."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return int(_load().ba_swa_fwd(ctypes.byref(problem), _ptr(q), _ptr(k), _ptr(v), _ptr(seq_offsets),
                                  int(window_tokens), _ptr(skip), _ptr(out), _ptr(lse), _ptr(workspace),
                                  int(workspace_bytes), _stream(stream)))


def ba_swa_bwd(problem, q, k, v, out, lse, dout, seq_offsets, window_tokens, skip, dq, dk, dv,
               workspace, workspace_bytes=None, stream=None) -> int:
    """Direct call of the sliding-window backward; returns its status code."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return int(_load().ba_swa_bwd(ctypes.byref(problem), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                  _ptr(dout), _ptr(seq_offsets), int(window_tokens), _ptr(skip),
                                  _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), int(workspace_bytes),
                                  _stream(stream)))


def _act(activation) -> int:
    if isinstance(activation, str):
        if activation not in _ACTS:
            raise ValueError(f"activation must be one of {sorted(_ACTS)}")
        return _ACTS[activation]
    return int(activation)


def ba_gdpa_workspace_size(problem: BAProblem, block: int, window: int) -> int:
    return int(_load().ba_gdpa_workspace_size(ctypes.byref(problem), int(block), int(window)))


def ba_gdpa_fwd(problem, activation, q, k, v, seq_offsets, block, window, out, workspace,
                workspace_bytes=None, stream=None) -> int:
    """Direct call of the generalized-attention forward; returns its status code."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return int(_load().ba_gdpa_fwd(ctypes.byref(problem), _act(activation), _ptr(q), _ptr(k), _ptr(v),
                                   _ptr(seq_offsets), int(block), int(window), _ptr(out), _ptr(workspace),
                                   int(workspace_bytes), _stream(stream)))


def ba_gdpa_bwd(problem, activation, q, k, v, dout, seq_offsets, block, window, dq, dk, dv, workspace,
                workspace_bytes=None, stream=None) -> int:
    """Direct call of the generalized-attention backward; returns its status code."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return int(_load().ba_gdpa_bwd(ctypes.byref(problem), _act(activation), _ptr(q), _ptr(k), _ptr(v),
                                   _ptr(dout), _ptr(seq_offsets), int(block), int(window), _ptr(dq), _ptr(dk),
                                   _ptr(dv), _ptr(workspace), int(workspace_bytes), _stream(stream)))


def gdpa_fwd(q, k, v, seq_offsets, block, window, activation="gelu", out=None, workspace=None, stream=None):
    """Generalized dot-product attention (activation in place of the softmax,
    block rule, no normalisation): allocates out (and a workspace) with torch
    and runs ba_gdpa_fwd."""
    _check_inputs(q, k, v, seq_offsets)
    prob = make_problem(q, seq_offsets)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = workspace_for(ba_gdpa_workspace_size(prob, block, window), q.device)
    st = ba_gdpa_fwd(prob, activation, q, k, v, seq_offsets, block, window, out, workspace, stream=stream)
    if st != BA_OK:
        raise BAError(st, "ba_gdpa_fwd")
    return out


def gdpa_bwd(q, k, v, dout, seq_offsets, block, window, activation="gelu", dq=None, dk=None, dv=None,
             workspace=None, stream=None):
    """Gradients of gdpa_fwd: allocates dq/dk/dv (and a workspace) with torch and runs ba_gdpa_bwd."""
    _check_inputs(q, k, v, seq_offsets)
    prob = make_problem(q, seq_offsets)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    if workspace is None:
        workspace = workspace_for(ba_gdpa_workspace_size(prob, block, window), q.device)
    st = ba_gdpa_bwd(prob, activation, q, k, v, dout, seq_offsets, block, window, dq, dk, dv, workspace,
                     stream=stream)
    if st != BA_OK:
        raise BAError(st, "ba_gdpa_bwd")
    return dq, dk, dv


def ba_gdpa_cross_workspace_size(problem: BAProblem, kv_total_tokens: int) -> int:
    return int(_load().ba_gdpa_cross_workspace_size(ctypes.byref(problem), int(kv_total_tokens)))


def ba_gdpa_cross_fwd(problem, kv_total_tokens, activation, q, k, v, q_offsets, kv_offsets, out, workspace,
                      workspace_bytes=None, stream=None) -> int:
    """Direct call of the cross-attention GDPA forward; returns its status code."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return int(_load().ba_gdpa_cross_fwd(ctypes.byref(problem), int(kv_total_tokens), _act(activation), _ptr(q),
                                         _ptr(k), _ptr(v), _ptr(q_offsets), _ptr(kv_offsets), _ptr(out),
                                         _ptr(workspace), int(workspace_bytes), _stream(stream)))


def ba_gdpa_cross_bwd(problem, kv_total_tokens, activation, q, k, v, dout, q_offsets, kv_offsets, dq, dk, dv,
                      workspace, workspace_bytes=None, stream=None) -> int:
    """Direct call of the cross-attention GDPA backward; returns its status code."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return int(_load().ba_gdpa_cross_bwd(ctypes.byref(problem), int(kv_total_tokens), _act(activation), _ptr(q),
                                         _ptr(k), _ptr(v), _ptr(dout), _ptr(q_offsets), _ptr(kv_offsets),
                                         _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), int(workspace_bytes),
                                         _stream(stream)))


def _check_cross(q, k, v, q_offsets, kv_offsets):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != q.dtype or t.dim() != 3:
            raise ValueError(f"{name} must be a contiguous CUDA tensor like q")
    if k.shape != v.shape or k.shape[1:] != q.shape[1:]:
        raise ValueError("k and v must be [kv_total_tokens, heads, head_dim] like q's heads and head_dim")
    for name, t in (("q_offsets", q_offsets), ("kv_offsets", kv_offsets)):
        if t.dtype != torch.int32 or not t.is_cuda:
            raise ValueError(f"{name} must be an int32 CUDA tensor")
    if q_offsets.numel() != kv_offsets.numel():
        raise ValueError("q_offsets and kv_offsets must describe the same examples")


def gdpa_cross_fwd(q, k, v, q_offsets, kv_offsets, activation="gelu", out=None, workspace=None, stream=None):
    """Cross-attention GDPA: example b's queries see every key of its own
    key/value set (no mask). Allocates out (and a workspace) with torch and
    runs ba_gdpa_cross_fwd."""
    _check_cross(q, k, v, q_offsets, kv_offsets)
    prob = make_problem(q, q_offsets)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = workspace_for(ba_gdpa_cross_workspace_size(prob, k.shape[0]), q.device)
    st = ba_gdpa_cross_fwd(prob, k.shape[0], activation, q, k, v, q_offsets, kv_offsets, out, workspace,
                           stream=stream)
    if st != BA_OK:
        raise BAError(st, "ba_gdpa_cross_fwd")
    return out


def gdpa_cross_bwd(q, k, v, dout, q_offsets, kv_offsets, activation="gelu", dq=None, dk=None, dv=None,
                   workspace=None, stream=None):
    """Gradients of gdpa_cross_fwd (ba_gdpa_cross_bwd)."""
    _check_cross(q, k, v, q_offsets, kv_offsets)
    prob = make_problem(q, q_offsets)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = workspace_for(ba_gdpa_cross_workspace_size(prob, k.shape[0]), q.device)
    st = ba_gdpa_cross_bwd(prob, k.shape[0], activation, q, k, v, dout, q_offsets, kv_offsets, dq, dk, dv,
                           workspace, stream=stream)
    if st != BA_OK:
        raise BAError(st, "ba_gdpa_cross_bwd")
    return dq, dk, dv


def ba_mx_quantize(x, elements, scales, stream=None) -> int:
    """Direct call of the MX (E4M3 / E8M0) quantisation of x [rows, heads, head_dim] bf16."""
    rows, heads, head_dim = x.shape
    return int(_load().ba_mx_quantize(_ptr(x), int(rows), int(heads), int(head_dim), _ptr(elements),
                                      _ptr(scales), _stream(stream)))


def mx_quantize(x, stream=None):
    """MX quantisation of a bf16 CUDA tensor [rows, heads, head_dim]: returns
    (elements uint8 [rows, heads, head_dim] holding E4M3 codes, scales uint8
    [rows, heads rounded up to 4, head_dim / 32] holding E8M0 codes)."""
    rows, heads, head_dim = x.shape
    elements = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    scales = torch.zeros((rows, (heads + 3) // 4 * 4, head_dim // 32), dtype=torch.uint8, device=x.device)
    st = ba_mx_quantize(x, elements, scales, stream)
    if st != BA_OK:
        raise BAError(st, "ba_mx_quantize")
    return elements, scales


def ba_mx_fwd_workspace_size(problem: BAProblem, block: int, window: int) -> int:
    return int(_load().ba_mx_fwd_workspace_size(ctypes.byref(problem), int(block), int(window)))


def ba_mx_fwd(problem, q, k, v, seq_offsets, block, window, skip, out, lse, workspace, workspace_bytes=None,
              stream=None) -> int:
    """Direct call of the MXFP8-operand forward; returns its status code."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return int(_load().ba_mx_fwd(ctypes.byref(problem), _ptr(q), _ptr(k), _ptr(v), _ptr(seq_offsets), int(block),
                                 int(window), _ptr(skip), _ptr(out), _ptr(lse), _ptr(workspace),
                                 int(workspace_bytes), _stream(stream)))


def mx_block_attention_fwd(q, k, v, seq_offsets, block, window, skip=None, out=None, lse=None, workspace=None,
                           stream=None):
    """Block attention with MXFP8 Q and K in the score product (ba_mx_fwd);
    allocates out/lse (and a workspace) with torch."""
    _check_inputs(q, k, v, seq_offsets)
    prob = make_problem(q, seq_offsets)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((q.shape[1], q.shape[0]), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = workspace_for(ba_mx_fwd_workspace_size(prob, block, window), q.device)
    st = ba_mx_fwd(prob, q, k, v, seq_offsets, block, window, skip, out, lse, workspace, stream=stream)
    if st != BA_OK:
        raise BAError(st, "ba_mx_fwd")
    return out, lse


def ba_mx_bwd_workspace_size(problem: BAProblem, block: int, window: int) -> int:
    return int(_load().ba_mx_bwd_workspace_size(ctypes.byref(problem), int(block), int(window)))


def ba_mx_bwd(problem, q, k, v, out, lse, dout, seq_offsets, block, window, skip, dq, dk, dv,
              workspace, workspace_bytes=None, stream=None) -> int:
    """Direct call of the MXFP8-operand backward; returns its status code."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return int(_load().ba_mx_bwd(ctypes.byref(problem), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                 _ptr(dout), _ptr(seq_offsets), int(block), int(window), _ptr(skip),
                                 _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), int(workspace_bytes),
                                 _stream(stream)))


def mx_block_attention_bwd(q, k, v, out, lse, dout, seq_offsets, block, window, skip=None,
                           dq=None, dk=None, dv=None, workspace=None, stream=None):
    """The backward of mx_block_attention_fwd (ba_mx_bwd); allocates dq/dk/dv
    (and a workspace) with torch."""
    _check_inputs(q, k, v, seq_offsets)
    prob = make_problem(q, seq_offsets)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    if workspace is None:
        workspace = workspace_for(ba_mx_bwd_workspace_size(prob, block, window), q.device)
    st = ba_mx_bwd(prob, q, k, v, out, lse, dout, seq_offsets, block, window, skip, dq, dk, dv, workspace,
                   stream=stream)
    if st != BA_OK:
        raise BAError(st, "ba_mx_bwd")
    return dq, dk, dv


def make_rope(cos, sin, q_rot=None, k_rot=None) -> BARope:
    """Rotary tables (float32 CUDA tensors [rows, head_dim / 2]) as the C
    struct, with optional caller buffers for the rotated q and k."""
    for name, t in (("cos", cos), ("sin", sin)):
        if not isinstance(t, int) and (t.dtype != torch.float32 or t.dim() != 2 or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous float32 [rows, head_dim / 2] tensor")
    rows = cos.shape[0] if not isinstance(cos, int) else 0
    return BARope(_ptr(cos), _ptr(sin), int(rows), _ptr(q_rot), _ptr(k_rot))


def ba_rope_fwd_workspace_size(problem: BAProblem, block: int, window: int) -> int:
    return int(_load().ba_rope_fwd_workspace_size(ctypes.byref(problem), int(block), int(window)))


def ba_rope_bwd_workspace_size(problem: BAProblem, block: int, window: int) -> int:
    return int(_load().ba_rope_bwd_workspace_size(ctypes.byref(problem), int(block), int(window)))


def ba_rope_fwd(problem, rope, q, k, v, seq_offsets, block, window, skip, out, lse, workspace,
                workspace_bytes=None, stream=None) -> int:
    """Direct call of the rotary forward (rope: BARope or None); returns its status code."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return int(_load().ba_rope_fwd(ctypes.byref(problem), ctypes.byref(rope) if rope is not None else None,
                                   _ptr(q), _ptr(k), _ptr(v), _ptr(seq_offsets), int(block), int(window),
                                   _ptr(skip), _ptr(out), _ptr(lse), _ptr(workspace), int(workspace_bytes),
                                   _stream(stream)))


def ba_rope_bwd(problem, rope, q, k, v, out, lse, dout, seq_offsets, block, window, skip, dq, dk, dv,
                workspace, workspace_bytes=None, stream=None) -> int:
    """Direct call of the rotary backward; returns its status code."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return int(_load().ba_rope_bwd(ctypes.byref(problem), ctypes.byref(rope) if rope is not None else None,
                                   _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout),
                                   _ptr(seq_offsets), int(block), int(window), _ptr(skip), _ptr(dq), _ptr(dk),
                                   _ptr(dv), _ptr(workspace), int(workspace_bytes), _stream(stream)))


def ba_set_profile_events(which: int, start=None, stop=None) -> int:
    """Record torch.cuda.Event ``start``/``stop`` around one kernel of every
    later call from this thread: 0 the forward attention kernel, 1 the
    backward dQ kernel, 2 the backward dK/dV kernel.
    The events must already exist on the device (torch creates an event on
    its first ``record``)."""
    s = start.cuda_event if start is not None else None
    e = stop.cuda_event if stop is not None else None
    if (start is not None and not s) or (stop is not None and not e):
        raise ValueError("record each event once before handing it to the library")
    return int(_load().ba_set_profile_events(int(which), s, e))


def ba_selftest_wait_timeout(workspace, limit_us: int, workspace_bytes=None, stream=None) -> int:
    """Launch the bounded-wait self-test (a wait that must time out); returns its status code."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return int(_load().ba_selftest_wait_timeout(_ptr(workspace), int(workspace_bytes), int(limit_us),
                                                _stream(stream)))


def ba_selftest_exp2(x, y, stream=None) -> int:
    """y = the kernels' FMA-pipe 2^x for float32 CUDA tensors x, y of equal size."""
    if x.dtype != torch.float32 or y.dtype != torch.float32 or x.numel() != y.numel():
        raise ValueError("x and y must be float32 tensors of equal size")
    return int(_load().ba_selftest_exp2(_ptr(x), _ptr(y), int(x.numel()), _stream(stream)))


def ba_selftest_activation(act, x, y, dy, stream=None) -> int:
    """y = act(x), dy = act'(x) through the generalized attention's device
    functions (act: BA_ACT_GELU or BA_ACT_SILU), float32 CUDA tensors of equal size."""
    if any(t.dtype != torch.float32 or t.numel() != x.numel() for t in (x, y, dy)):
        raise ValueError("x, y and dy must be float32 tensors of equal size")
    return int(_load().ba_selftest_activation(int(act), _ptr(x), _ptr(y), _ptr(dy), int(x.numel()),
                                              _stream(stream)))


def ba_device_status(workspace, stream=None) -> int:
    return int(_load().ba_device_status(_ptr(workspace), _stream(stream)))


def _check_inputs(q, k, v, seq_offsets):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError(f"{name} must match q in shape and dtype")
    if seq_offsets.dtype != torch.int32 or not seq_offsets.is_cuda:
        raise ValueError("seq_offsets must be an int32 CUDA tensor")


def workspace_for(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns 512-byte-aligned blocks
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def block_attention_fwd(q, k, v, seq_offsets, block, window, skip=None, out=None, lse=None,
                        workspace=None, stream=None):
    """Allocates out/lse (and a workspace) with torch and runs ba_fwd."""
    _check_inputs(q, k, v, seq_offsets)
    prob = make_problem(q, seq_offsets)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((q.shape[1], q.shape[0]), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = workspace_for(ba_fwd_workspace_size(prob, block, window), q.device)
    st = ba_fwd(prob, q, k, v, seq_offsets, block, window, skip, out, lse, workspace, stream=stream)
    if st != BA_OK:
        raise BAError(st, "ba_fwd")
    return out, lse


def block_attention_bwd(q, k, v, out, lse, dout, seq_offsets, block, window, skip=None,
                        dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Allocates dq/dk/dv (and a workspace) with torch and runs ba_bwd."""
    _check_inputs(q, k, v, seq_offsets)
    prob = make_problem(q, seq_offsets)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    if workspace is None:
        workspace = workspace_for(ba_bwd_workspace_size(prob, block, window), q.device)
    st = ba_bwd(prob, q, k, v, out, lse, dout, seq_offsets, block, window, skip, dq, dk, dv,
                workspace, stream=stream)
    if st != BA_OK:
        raise BAError(st, "ba_bwd")
    return dq, dk, dv


def sliding_window_attention_fwd(q, k, v, seq_offsets, window_tokens, skip=None, out=None, lse=None,
                                 workspace=None, stream=None):
    """Allocates out/lse (and a workspace) with torch and runs ba_swa_fwd:
    query i sees keys i - window_tokens < j <= i of its example."""
    _check_inputs(q, k, v, seq_offsets)
    prob = make_problem(q, seq_offsets)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((q.shape[1], q.shape[0]), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = workspace_for(ba_swa_fwd_workspace_size(prob, window_tokens), q.device)
    st = ba_swa_fwd(prob, q, k, v, seq_offsets, window_tokens, skip, out, lse, workspace, stream=stream)
    if st != BA_OK:
        raise BAError(st, "ba_swa_fwd")
    return out, lse


def sliding_window_attention_bwd(q, k, v, out, lse, dout, seq_offsets, window_tokens, skip=None,
                                 dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Allocates dq/dk/dv (and a workspace) with torch and runs ba_swa_bwd."""
    _check_inputs(q, k, v, seq_offsets)
    prob = make_problem(q, seq_offsets)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    if workspace is None:
        workspace = workspace_for(ba_swa_bwd_workspace_size(prob, window_tokens), q.device)
    st = ba_swa_bwd(prob, q, k, v, out, lse, dout, seq_offsets, window_tokens, skip, dq, dk, dv,
                    workspace, stream=stream)
    if st != BA_OK:
        raise BAError(st, "ba_swa_bwd")
    return dq, dk, dv


def _check_tables(cos, sin, q):
    for name, t in (("cos", cos), ("sin", sin)):
        if not t.is_cuda or t.dtype != torch.float32 or t.dim() != 2 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous float32 CUDA tensor [rows, head_dim / 2]")
        if t.shape[1] != q.shape[2] // 2 or t.shape != cos.shape:
            raise ValueError("cos and sin must both be [rows, head_dim / 2]")


def _check_rotated(q_rot, k_rot, q):
    if (q_rot is None) != (k_rot is None):
        raise ValueError("pass both q_rot and k_rot, or neither")
    for name, t in (("q_rot", q_rot), ("k_rot", k_rot)):
        if t is not None and (not t.is_cuda or not t.is_contiguous() or t.shape != q.shape or t.dtype != q.dtype):
            raise ValueError(f"{name} must be a contiguous CUDA tensor like q")


def rope_block_attention_fwd(q, k, v, seq_offsets, block, window, cos, sin, skip=None, out=None, lse=None,
                             workspace=None, q_rot=None, k_rot=None, stream=None):
    """Rotary embedding on q and k (tables cos, sin [rows, head_dim / 2];
    rows must cover the longest example), then block attention: ba_rope_fwd.
    Allocates out/lse (and a workspace) with torch. q_rot / k_rot: buffers
    like q that receive the rotated q and k, to hand to the backward."""
    _check_inputs(q, k, v, seq_offsets)
    _check_tables(cos, sin, q)
    _check_rotated(q_rot, k_rot, q)
    prob = make_problem(q, seq_offsets)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((q.shape[1], q.shape[0]), dtype=torch.float32, device=q.device)
    if workspace is None:
        need = (ba_fwd_workspace_size if q_rot is not None else ba_rope_fwd_workspace_size)(prob, block, window)
        workspace = workspace_for(need, q.device)
    st = ba_rope_fwd(prob, make_rope(cos, sin, q_rot, k_rot), q, k, v, seq_offsets, block, window, skip, out,
                     lse, workspace, stream=stream)
    if st != BA_OK:
        raise BAError(st, "ba_rope_fwd")
    return out, lse


def rope_block_attention_bwd(q, k, v, out, lse, dout, seq_offsets, block, window, cos, sin, skip=None,
                             dq=None, dk=None, dv=None, workspace=None, q_rot=None, k_rot=None, stream=None):
    """Gradients of rope_block_attention_fwd with respect to the unrotated q,
    k and v: ba_rope_bwd. Allocates dq/dk/dv (and a workspace) with torch.
    q_rot / k_rot: the forward's rotated copies (then no rotation pass runs)."""
    _check_inputs(q, k, v, seq_offsets)
    _check_tables(cos, sin, q)
    _check_rotated(q_rot, k_rot, q)
    prob = make_problem(q, seq_offsets)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    if workspace is None:
        need = (ba_bwd_workspace_size if q_rot is not None else ba_rope_bwd_workspace_size)(prob, block, window)
        workspace = workspace_for(need, q.device)
    st = ba_rope_bwd(prob, make_rope(cos, sin, q_rot, k_rot), q, k, v, out, lse, dout, seq_offsets, block,
                     window, skip, dq, dk, dv, workspace, stream=stream)
    if st != BA_OK:
        raise BAError(st, "ba_rope_bwd")
    return dq, dk, dv
