"""Python binding of libkda, the B200 (sm_100a) Kimi Delta Attention hot path.

The names mirror the C ABI of include/kda.h.  This module only marshals
arguments: it checks shapes, allocates outputs with torch when the caller
does not pass them, and hands raw device pointers and the current CUDA stream
to the library.  Every arithmetic step runs in the library's kernels; there is
no CPU or PyTorch fallback, and a missing libkda.so is an error.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["kda_chunk_fwd", "kda_recurrent_fwd", "kda_recurrent_bwd", "kda_chunk_fwd_noalloc", "kda_chunk_fwd_workspace_size", "kda_decode_step", "kda_selftest_bounded_wait", "kda_status_str", "library_path", "load_library",
           "KDAError", "KDA_F32", "KDA_BF16", "KDA_GATE_CHANNEL", "KDA_GATE_SCALAR",
           "KDA_GATE_NONE", "KDA_DEV_BAD_SEQLENS", "KDA_DEV_TIMEOUT", "Shape"]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libkda.so")

KDA_F32, KDA_BF16 = 0, 1
KDA_GATE_CHANNEL, KDA_GATE_SCALAR, KDA_GATE_NONE = 0, 1, 2
KDA_DEV_BAD_SEQLENS, KDA_DEV_TIMEOUT = 1, 2
_STATUS = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED",
           3: "KDA_ERR_MISALIGNED", 4: "KDA_ERR_CUDA", 5: "KDA_ERR_TIMEOUT", 6: "KDA_ERR_TOO_LARGE"}


class KDAError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {_STATUS.get(status, status)} ({kda_status_str(status)})")
        self.status = status


class Shape(ctypes.Structure):
    """kda_shape_t (qk_heads = 0: one query/key head per value head)."""
    _fields_ = [("B", ctypes.c_int32), ("T", ctypes.c_int32), ("H", ctypes.c_int32),
                ("d_k", ctypes.c_int32), ("d_v", ctypes.c_int32), ("num_seqs", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("gate", ctypes.c_int32), ("chunk", ctypes.c_int32),
                ("dev_status", ctypes.c_void_p), ("qk_heads", ctypes.c_int32)]


_lib = None


def library_path() -> str:
    return _LIB_PATH


def load_library(path: str | None = None):
    """Load libkda.so (built in-tree by __graft_entry__.build()).  Raises if it is missing."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or _LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"libkda.so not found at {p}: build it with "
                           "`python -m kimi_delta_attention_22_b200.build`")
    lib = ctypes.CDLL(p)
    P = ctypes.c_void_p
    lib.kda_chunk_fwd.argtypes = [ctypes.POINTER(Shape), P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t,
                                  P]
    lib.kda_chunk_fwd_noalloc.argtypes = [ctypes.POINTER(Shape), P, P, P, P, P, P, P, P, P, P]
    lib.kda_chunk_fwd_noalloc.restype = ctypes.c_int
    lib.kda_chunk_fwd_workspace_size.argtypes = [ctypes.POINTER(Shape), ctypes.c_int]
    lib.kda_chunk_fwd_workspace_size.restype = ctypes.c_size_t
    lib.kda_chunk_fwd.restype = ctypes.c_int
    lib.kda_decode_step.argtypes = [ctypes.POINTER(Shape), P, P, P, P, P, P, P, P]
    lib.kda_recurrent_fwd.argtypes = [ctypes.POINTER(Shape), P, P, P, P, P, P, P, P]
    lib.kda_recurrent_fwd.restype = ctypes.c_int
    lib.kda_recurrent_bwd.argtypes = [ctypes.POINTER(Shape)] + [P] * 15 + [ctypes.c_size_t, P]
    lib.kda_recurrent_bwd.restype = ctypes.c_int
    lib.kda_chunk_bwd.argtypes = [ctypes.POINTER(Shape)] + [P] * 16 + [ctypes.c_size_t, P]
    lib.kda_chunk_bwd.restype = ctypes.c_int
    lib.kda_chunk_bwd_workspace_size.argtypes = [ctypes.POINTER(Shape), ctypes.c_int]
    lib.kda_chunk_bwd_workspace_size.restype = ctypes.c_size_t
    lib.kda_recurrent_bwd_workspace_size.argtypes = [ctypes.POINTER(Shape)]
    lib.kda_recurrent_bwd_workspace_size.restype = ctypes.c_size_t
    lib.kda_decode_step.restype = ctypes.c_int
    lib.kda_status_str.argtypes = [ctypes.c_int]
    lib.kda_status_str.restype = ctypes.c_char_p
    lib.kda_version.restype = ctypes.c_char_p
    lib.kda_selftest_bounded_wait.argtypes = [P, ctypes.c_uint32, ctypes.c_int32, P]
    lib.kda_selftest_bounded_wait.restype = ctypes.c_int
    if path is None:
        _lib = lib
    return lib


def kda_status_str(status: int) -> str:
    return load_library().kda_status_str(int(status)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(dt) -> int:
    if dt == torch.bfloat16:
        return KDA_BF16
    if dt == torch.float32:
        return KDA_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {dt}")


def _gate_code(g, q) -> int:
    if g is None:
        return KDA_GATE_NONE
    if g.dim() == q.dim():
        return KDA_GATE_CHANNEL
    if g.dim() == q.dim() - 1:
        return KDA_GATE_SCALAR
    raise ValueError(f"g has {g.dim()} dims; expected {q.dim()} (per channel) or {q.dim() - 1} (scalar)")


def _heads(q, v, lead: int):
    """(value heads H, query/key heads Hk) from q [.., Hk, d_k] and v [.., H, d_v]
    (`lead` leading dims before the head axis); H must be a multiple of Hk."""
    Hk, H = q.shape[lead], v.shape[lead]
    if v.shape[:lead] != q.shape[:lead] or Hk <= 0 or H % Hk != 0:
        raise ValueError(f"q/k heads ({Hk}) must divide the value heads of v ({H}) with equal leading dims")
    return H, Hk


def _check_cuda(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("libkda takes device tensors (copy host data to the GPU first)")
            if not t.is_contiguous():
                raise ValueError("libkda takes contiguous tensors")


def kda_chunk_fwd(q, k, v, g, beta, S0=None, cu_seqlens=None, chunk: int = 64, out=None,
                  S_T=None, want_state: bool = True, dev_status=None, workspace=True, lib=None):
    """Chunkwise KDA prefill (kda_chunk_fwd of include/kda.h).

    q, k [B,T,Hk,d_k]; v [B,T,H,d_v] (bf16 or fp32, same dtype); g [B,T,H,d_k]
    (per channel) | [B,T,H] (scalar) | None (no gate), fp32 log-decay;
    beta [B,T,H] fp32; S0 [N,H,d_v,d_k] fp32 or None; cu_seqlens int32 [N+1]
    with B == 1 for packed sequences.  H value heads, Hk query/key heads
    (H a multiple of Hk; value head h reads q/k head h // (H // Hk)).
    Returns (out, S_T); S_T is None when want_state is False and no S_T buffer
    is given.

    workspace: True allocates the tensor-core path's scratch with torch (when the
    shape takes a path that uses one), a uint8 CUDA tensor supplies it, and None /
    False passes no workspace, so that the library takes the scratch from the
    device's stream-ordered memory pool on the current stream.
    """
    _check_cuda(q, k, v, g, beta, S0, cu_seqlens, out, S_T, dev_status)
    B, T, Hk, Dk = q.shape
    H, _ = _heads(q, v, 2)
    Dv = v.shape[-1]
    N = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if k.shape != q.shape or beta.shape != v.shape[:3]:
        raise ValueError("shape mismatch among q, k, v, beta")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    if g is not None and g.dtype != torch.float32 or beta.dtype != torch.float32:
        raise TypeError("g and beta are float32")
    if cu_seqlens is not None and cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens is int32")
    if out is None:
        out = torch.empty_like(v)
    if S_T is None and want_state:
        S_T = torch.empty(N, H, Dv, Dk, dtype=torch.float32, device=q.device)
    sh = Shape(B, T, H, Dk, Dv, N, _dtype_code(q.dtype), _gate_code(g, q), int(chunk),
               None if dev_status is None else dev_status.data_ptr(), Hk)
    lib = lib or load_library()
    if isinstance(workspace, torch.Tensor):
        _check_cuda(workspace)
    if workspace is True:
        nbytes = lib.kda_chunk_fwd_workspace_size(ctypes.byref(sh), int(cu_seqlens is not None))
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device) if nbytes else None
    elif workspace is False:
        workspace = None
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.kda_chunk_fwd(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                           _ptr(S0), _ptr(cu_seqlens), _ptr(out), _ptr(S_T), _ptr(workspace),
                           ws_bytes, _stream_handle(q.device))
    if st != 0:
        raise KDAError(st, "kda_chunk_fwd")
    return out, S_T


def kda_chunk_fwd_noalloc(q, k, v, g, beta, S0=None, cu_seqlens=None, chunk: int = 64, out=None,
                          S_T=None, want_state: bool = True, dev_status=None, lib=None):
    """kda_chunk_fwd_noalloc of include/kda.h: the library's own static scratch
    instead of a workspace (arguments and results as kda_chunk_fwd)."""
    _check_cuda(q, k, v, g, beta, S0, cu_seqlens, out, S_T, dev_status)
    B, T, Hk, Dk = q.shape
    H, _ = _heads(q, v, 2)
    Dv = v.shape[-1]
    N = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty_like(v)
    if S_T is None and want_state:
        S_T = torch.empty(N, H, Dv, Dk, dtype=torch.float32, device=q.device)
    sh = Shape(B, T, H, Dk, Dv, N, _dtype_code(q.dtype), _gate_code(g, q), int(chunk),
               None if dev_status is None else dev_status.data_ptr(), Hk)
    lib = lib or load_library()
    st = lib.kda_chunk_fwd_noalloc(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                   _ptr(S0), _ptr(cu_seqlens), _ptr(out), _ptr(S_T),
                                   _stream_handle(q.device))
    if st != 0:
        raise KDAError(st, "kda_chunk_fwd_noalloc")
    return out, S_T


def kda_chunk_fwd_workspace_size(q, v, g=None, cu_seqlens=None, chunk: int = 64, lib=None) -> int:
    """Bytes of scratch the two-kernel schedule needs for these inputs (0: none)."""
    B, T, Hk, Dk = q.shape
    H, _ = _heads(q, v, 2)
    N = B if cu_seqlens is None else cu_seqlens.numel() - 1
    sh = Shape(B, T, H, Dk, v.shape[-1], N, _dtype_code(q.dtype), _gate_code(g, q), int(chunk), None, Hk)
    lib = lib or load_library()
    return int(lib.kda_chunk_fwd_workspace_size(ctypes.byref(sh), int(cu_seqlens is not None)))


def kda_decode_step(q, k, v, g, beta, S, out=None, lib=None):
    """One fused recurrent KDA token (kda_decode_step of include/kda.h).

    q, k [N,Hk,d_k]; v [N,H,d_v]; g [N,H,d_k] | [N,H] | None (fp32 log-decay);
    beta [N,H] fp32; S [N,H,d_v,d_k] fp32, updated in place.  Returns out [N,H,d_v].
    H value heads, Hk query/key heads (H a multiple of Hk).
    """
    _check_cuda(q, k, v, g, beta, S, out)
    N, Hk, Dk = q.shape
    H, _ = _heads(q, v, 1)
    Dv = v.shape[-1]
    if S.shape != (N, H, Dv, Dk) or S.dtype != torch.float32:
        raise ValueError("S must be float32 [N, H, d_v, d_k]")
    if out is None:
        out = torch.empty_like(v)
    sh = Shape(N, 1, H, Dk, Dv, N, _dtype_code(q.dtype), _gate_code(g, q), 0, None, Hk)
    lib = lib or load_library()
    st = lib.kda_decode_step(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                             _ptr(S), _ptr(out), _stream_handle(q.device))
    if st != 0:
        raise KDAError(st, "kda_decode_step")
    return out


def kda_recurrent_fwd(q, k, v, g, beta, S, out=None, lib=None):
    """Fused recurrent KDA over T tokens per sequence (kda_recurrent_fwd of include/kda.h).

    q, k [N,T,Hk,d_k]; v [N,T,H,d_v]; g [N,T,H,d_k] | [N,T,H] | None (fp32 log-decay);
    beta [N,T,H] fp32; S [N,H,d_v,d_k] fp32, read once and overwritten with the state
    after the T tokens.  Returns out [N,T,H,d_v].  H value heads, Hk query/key heads
    (H a multiple of Hk).
    """
    _check_cuda(q, k, v, g, beta, S, out)
    N, T, Hk, Dk = q.shape
    H, _ = _heads(q, v, 2)
    Dv = v.shape[-1]
    if S.shape != (N, H, Dv, Dk) or S.dtype != torch.float32:
        raise ValueError("S must be float32 [N, H, d_v, d_k]")
    if out is None:
        out = torch.empty_like(v)
    sh = Shape(N, T, H, Dk, Dv, N, _dtype_code(q.dtype), _gate_code(g, q), 0, None, Hk)
    lib = lib or load_library()
    st = lib.kda_recurrent_fwd(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                               _ptr(S), _ptr(out), _stream_handle(q.device))
    if st != 0:
        raise KDAError(st, "kda_recurrent_fwd")
    return out


def kda_recurrent_bwd(q, k, v, g, beta, S0, d_out, d_ST=None, want_dS0: bool = True, workspace=None,
                      lib=None):
    """Gradients of kda_recurrent_fwd (kda_recurrent_bwd of include/kda.h).

    Inputs as kda_recurrent_fwd, with S0 [N,H,d_v,d_k] fp32 or None (the state
    before the tokens; not modified), d_out [N,T,H,d_v] in the input dtype and
    d_ST [N,H,d_v,d_k] fp32 or None.  Returns a dict of fp32 tensors dq, dk
    [N,T,Hk,d_k], dv [N,T,H,d_v], dg (shape of g, or None), dbeta [N,T,H] and
    dS0 [N,H,d_v,d_k] (None unless want_dS0) for the loss
    sum(out * d_out) + sum(S_T * d_ST).
    """
    _check_cuda(q, k, v, g, beta, S0, d_out, d_ST)
    N, T, Hk, Dk = q.shape
    H, _ = _heads(q, v, 2)
    Dv = v.shape[-1]
    if d_out.shape != v.shape or d_out.dtype != v.dtype:
        raise ValueError("d_out must match v in shape and dtype")
    f32 = dict(dtype=torch.float32, device=q.device)
    dq = torch.empty(N, T, Hk, Dk, **f32)
    dk = torch.empty(N, T, Hk, Dk, **f32)
    dv = torch.empty(N, T, H, Dv, **f32)
    dg = None if g is None else torch.empty(g.shape, **f32)
    dbeta = torch.empty(N, T, H, **f32)
    dS0 = torch.empty(N, H, Dv, Dk, **f32) if want_dS0 else None
    sh = Shape(N, T, H, Dk, Dv, N, _dtype_code(q.dtype), _gate_code(g, q), 0, None, Hk)
    lib = lib or load_library()
    if workspace is None:
        nbytes = lib.kda_recurrent_bwd_workspace_size(ctypes.byref(sh))
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    _check_cuda(workspace)
    st = lib.kda_recurrent_bwd(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                               _ptr(d_out), _ptr(d_ST), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg), _ptr(dbeta),
                               _ptr(dS0), _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _stream_handle(q.device))
    if st != 0:
        raise KDAError(st, "kda_recurrent_bwd")
    return dict(dq=dq, dk=dk, dv=dv, dg=dg, dbeta=dbeta, dS0=dS0)


def kda_chunk_bwd(q, k, v, g, beta, S0, d_out, d_ST=None, cu_seqlens=None, chunk: int = 64,
                  want_dS0: bool = True, dev_status=None, workspace=True, lib=None):
    """Gradients of kda_chunk_fwd (kda_chunk_bwd of include/kda.h), chunkwise.

    Inputs as kda_chunk_fwd (bf16 q, k, v with d_k = d_v = 128, chunk 64; dense or
    packed through cu_seqlens), with d_out [B,T,H,d_v] bf16 and d_ST [N,H,d_v,d_k]
    fp32 or None.  Returns a dict of fp32 tensors dq, dk [B,T,Hk,d_k], dv
    [B,T,H,d_v], dg (shape of g, or None), dbeta [B,T,H] and dS0 [N,H,d_v,d_k]
    (None unless want_dS0) for the loss sum(out * d_out) + sum(S_T * d_ST).

    workspace: True allocates the scratch with torch, a uint8 CUDA tensor supplies
    it, None / False lets the library take it from the stream-ordered pool.
    """
    _check_cuda(q, k, v, g, beta, S0, d_out, d_ST, cu_seqlens, dev_status)
    B, T, Hk, Dk = q.shape
    H, _ = _heads(q, v, 2)
    Dv = v.shape[-1]
    N = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if d_out.shape != v.shape or d_out.dtype != v.dtype:
        raise ValueError("d_out must match v in shape and dtype")
    if cu_seqlens is not None and cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens is int32")
    f32 = dict(dtype=torch.float32, device=q.device)
    dq = torch.empty(B, T, Hk, Dk, **f32)
    dk = torch.empty(B, T, Hk, Dk, **f32)
    dv = torch.empty(B, T, H, Dv, **f32)
    dg = None if g is None else torch.empty(g.shape, **f32)
    dbeta = torch.empty(B, T, H, **f32)
    dS0 = torch.empty(N, H, Dv, Dk, **f32) if want_dS0 else None
    sh = Shape(B, T, H, Dk, Dv, N, _dtype_code(q.dtype), _gate_code(g, q), int(chunk),
               None if dev_status is None else dev_status.data_ptr(), Hk)
    lib = lib or load_library()
    if isinstance(workspace, torch.Tensor):
        _check_cuda(workspace)
    if workspace is True:
        nbytes = lib.kda_chunk_bwd_workspace_size(ctypes.byref(sh), int(cu_seqlens is not None))
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device) if nbytes else None
    elif workspace is False:
        workspace = None
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.kda_chunk_bwd(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                           _ptr(cu_seqlens), _ptr(d_out), _ptr(d_ST), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg),
                           _ptr(dbeta), _ptr(dS0), _ptr(workspace), ws_bytes, _stream_handle(q.device))
    if st != 0:
        raise KDAError(st, "kda_chunk_bwd")
    return dict(dq=dq, dk=dk, dv=dv, dg=dg, dbeta=dbeta, dS0=dS0)


def kda_selftest_bounded_wait(dev_status: torch.Tensor, budget_us: int, complete: bool = False,
                              lib=None) -> None:
    """kda_selftest_bounded_wait: one CTA takes the kernels' bounded mbarrier wait
    (budget_us microseconds) on a barrier that never completes (complete=False;
    KDA_DEV_TIMEOUT is ORed into dev_status) or completes at once (complete=True;
    dev_status untouched).  dev_status: int32 device tensor; read it after a sync."""
    _check_cuda(dev_status)
    if dev_status.dtype != torch.int32 or dev_status.numel() < 1:
        raise ValueError("dev_status must be an int32 device tensor")
    lib = lib or load_library()
    st = lib.kda_selftest_bounded_wait(_ptr(dev_status), int(budget_us), int(bool(complete)),
                                       _stream_handle(dev_status.device))
    if st != 0:
        raise KDAError(st, "kda_selftest_bounded_wait")
