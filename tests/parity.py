"""Helpers shared by the GPU parity tests: run the library and the float64
oracle on the same seeded inputs and compare element by element."""
from __future__ import annotations

import numpy as np
import torch

import kimi_delta_attention_22_b200 as kda
import oracle
from kimi_delta_attention_22_b200 import inputs

# Tolerances (see the readings of the pages): fp32 mode is compared by the
# maximum absolute error; bf16-input/fp32-state mode by the maximum absolute
# error divided by the RMS of the oracle's tensor, per tensor.
TOL_F32_ABS = 1e-4
TOL_BF16_REL = 2e-2


def to_dev(d, dev="cuda"):
    return {k: (None if v is None else v.to(dev)) for k, v in d.items()}


def err(got, ref, mode):
    got = got.detach().cpu().double().numpy() if hasattr(got, "detach") else np.asarray(got)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in the GPU result"
    if got.size == 0:
        return 0.0
    e = float(np.max(np.abs(got - ref)))
    if mode == "f32":
        return e
    rms = float(np.sqrt(np.mean(ref ** 2)))
    return e / max(rms, 1e-30)


def check(got, ref, mode, what):
    e = err(got, ref, mode)
    tol = TOL_F32_ABS if mode == "f32" else TOL_BF16_REL
    assert e <= tol, f"{what}: error {e:.3e} > {tol:.1e} ({'max abs' if mode == 'f32' else 'max abs / rms'})"
    return e


def run_chunk(d, chunk, want_state=True, cu=None):
    on = to_dev(d)
    out, ST = kda.kda_chunk_fwd(on["q"], on["k"], on["v"], on["g"], on["beta"], S0=on["S0"],
                                cu_seqlens=on.get("cu_seqlens") if cu is None else cu.cuda(),
                                chunk=chunk, want_state=want_state)
    torch.cuda.synchronize()
    return out, ST


def oracle_chunk(d, gate):
    return oracle.forward(d["q"], d["k"], d["v"], d["g"], d["beta"], S0=d["S0"],
                          cu_seqlens=d.get("cu_seqlens"), gate=gate)


def gate_of(d):
    g, q = d["g"], d["q"]
    if g is None:
        return "none"
    return "channel" if g.dim() == q.dim() else "scalar"


def sampled_pairs_oracle(d, pairs, gate):
    """Oracle on selected (sequence, head) pairs of a dense batch only.
    Returns {(n, h): (out [T, d_v], S_T [d_v, d_k])}."""
    res = {}
    for n, h in pairs:
        sl = lambda t: None if t is None else t[n:n + 1, :, h:h + 1]
        s0 = None if d["S0"] is None else d["S0"][n:n + 1, h:h + 1]
        o, s = oracle.forward(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["g"]), sl(d["beta"]),
                              S0=s0, gate=gate)
        res[(n, h)] = (o[0, :, 0], s[0, 0])
    return res


def sampled_varlen_oracle(d, pairs, gate):
    """Oracle on selected (sequence, head) pairs of a packed batch."""
    cu = d["cu_seqlens"].cpu().numpy()
    res = {}
    for n, h in pairs:
        a, b = int(cu[n]), int(cu[n + 1])
        sl = lambda t: None if t is None else t[:, a:b, h:h + 1]
        s0 = None if d["S0"] is None else d["S0"][n:n + 1, h:h + 1]
        o, s = oracle.forward(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["g"]), sl(d["beta"]),
                              S0=s0, gate=gate)
        res[(n, h)] = (o[0, :, 0], s[0, 0])
    return res
