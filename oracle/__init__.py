"""Float64 CPU oracle for the Kimi Delta Attention (KDA) recurrence.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s cpu_baseline / reference arm may import this package; the
library's product path never does, and the two share no code.

What it computes is the five-step KDA state update of "You could have come up
with Kimi Delta Attention" (the equations at the top of the article; the same
steps in the GeekNews summary, section "Kimi Delta Attention: per-channel
decay"), token by token in float64, in ``kda_oracle.c``.  This module only
marshals numpy arrays into that C function.

``chunkwise_mirror`` (a separate module) restates the chunkwise form in numpy
float64 for debugging; it is checked against this oracle, never the reverse.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_lib = None

GATE_CHANNEL, GATE_SCALAR, GATE_NONE = 0, 1, 2
_GATE_NAMES = {"channel": GATE_CHANNEL, "scalar": GATE_SCALAR, "none": GATE_NONE}


def build(force: bool = False) -> str:
    """Compile kda_oracle.c into libkda_oracle.so beside it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def bind(path: str):
    """Load a compiled oracle library and declare its C signatures."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    lib.kda_oracle_forward.argtypes = [ctypes.c_int, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, P, P, P, P, P, P, P, P,
                                       ctypes.c_int]
    lib.kda_oracle_forward.restype = ctypes.c_int
    lib.kda_oracle_max_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = bind(_LIB_PATH)
    return _lib


def max_threads() -> int:
    return int(_load().kda_oracle_max_threads())


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: upcast exactly (bf16/fp32 -> fp64)
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def forward(q, k, v, g, beta, S0=None, cu_seqlens=None, gate="channel", want_state=True,
            nthreads: int = 0, lib=None):
    """Run the float64 KDA recurrence.

    Dense layout (cu_seqlens None): q,k [B,T,Hk,dk]; v [B,T,H,dv]; g [B,T,H,dk]
    (channel) / [B,T,H] (scalar) / None (none); beta [B,T,H]; S0 [B,H,dv,dk] or
    None.  Varlen layout: leading batch of 1 (or none), cu_seqlens [N+1] offsets
    into the packed token axis; S0 [N,H,dv,dk].  H is the number of value heads
    and a multiple of Hk: value head h reads query/key head h // (H // Hk)
    (Hk == H is the plain one-to-one case).

    Returns (out [same lead shape as v], S_T [num_seqs,H,dv,dk] or None), float64.
    Inputs are converted to float64 exactly (bf16 and fp32 both embed in fp64).
    """
    gate_mode = _GATE_NAMES[gate] if isinstance(gate, str) else int(gate)
    q, k, v, g, beta, S0 = (_f64(a) for a in (q, k, v, g, beta, S0))
    lead = v.shape[:-2]
    H, Hk, dk, dv = v.shape[-2], q.shape[-2], q.shape[-1], v.shape[-1]
    if k.shape != q.shape or H % Hk != 0:
        raise ValueError(f"q/k heads {q.shape[-2]} must divide the value heads {H}")
    if cu_seqlens is None:
        B, T = (1, lead[0]) if len(lead) == 1 else lead
        starts = np.arange(B, dtype=np.int64) * T
        lens = np.full(B, T, dtype=np.int64)
    else:
        cu = np.asarray(cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
                        dtype=np.int64).reshape(-1)
        starts = np.ascontiguousarray(cu[:-1])
        lens = np.ascontiguousarray(cu[1:] - cu[:-1])
    N = len(starts)
    rows = int(np.prod(lead))
    if gate_mode == GATE_NONE:
        g = None
    out = np.zeros(v.shape, dtype=np.float64)
    ST = np.zeros((N, H, dv, dk), dtype=np.float64) if want_state else None
    if S0 is not None and S0.shape != (N, H, dv, dk):
        raise ValueError(f"S0 shape {S0.shape} != {(N, H, dv, dk)}")
    if lens.size and int((starts + lens).max()) > rows:
        raise ValueError("sequence extends past the token axis")
    rc = (lib or _load()).kda_oracle_forward(N, _ptr(starts), _ptr(lens), H, Hk, dk, dv, gate_mode,
                                    _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                                    _ptr(out), _ptr(ST), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_forward failed with code {rc}")
    return out, ST


def decode_step(q, k, v, g, beta, S, gate="channel", lib=None):
    """One recurrent token per (sequence, head): q,k [N,H,dk], v [N,H,dv],
    g [N,H,dk] / [N,H] / None, beta [N,H], S [N,H,dv,dk].  Returns (out, S_new)."""
    q, k, v, g, beta, S = (_f64(a) for a in (q, k, v, g, beta, S))
    out, ST = forward(q[:, None], k[:, None], v[:, None], None if g is None else g[:, None],
                      beta[:, None], S0=S, gate=gate, lib=lib)
    return out[:, 0], ST
