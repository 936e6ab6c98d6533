"""Helpers shared by the GPU parity tests: run the library and the float64
oracle on the same seeded inputs and compare element by element."""
from __future__ import annotations

import numpy as np
import torch

import kimi_delta_attention_22_b200 as kda
import oracle
from kimi_delta_attention_22_b200 import inputs

# Tolerances (see the readings of the pages).  fp32 mode: the maximum
# absolute error, max |gpu - oracle| <= 1e-4.  bf16-input/fp32-state mode:
# the error relative to the RMS of the oracle's tensor, per tensor, element by
# element: max |gpu - oracle| / rms(oracle) <= 2e-2, where for a tensor the
# library stores in bf16 each element may also differ by the rounding of the
# stored result, q |oracle| with q = 2^-8 (half a bf16 ulp, relative): rounding
# the returned value is not an arithmetic error of the path.  fp32 tensors
# (the final state) get no allowance.  The RMS ratio is reported beside it.
TOL_F32_ABS = 1e-4
TOL_BF16_REL = 2e-2
BF16_HALF_ULP = 2.0 ** -8


def to_dev(d, dev="cuda"):
    return {k: (None if v is None else v.to(dev)) for k, v in d.items()}


def err(got, ref, mode, stored_bf16=None):
    """Returns the error figure compared against TOL_F32_ABS (fp32 mode: max abs)
    or TOL_BF16_REL (bf16 mode: the worst element-wise excess over the stored-result
    rounding allowance, relative to rms(oracle); never below the RMS ratio)."""
    if stored_bf16 is None:
        stored_bf16 = hasattr(got, "dtype") and got.dtype == torch.bfloat16
    got = got.detach().cpu().double().numpy() if hasattr(got, "detach") else np.asarray(got)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in the GPU result"
    if got.size == 0:
        return 0.0
    d = np.abs(got - ref)
    if mode == "f32":
        return float(np.max(d))
    rms = max(float(np.sqrt(np.mean(ref ** 2))), 1e-30)
    # "both": two independently rounded bf16 results may differ by a full ulp
    q = 2 * BF16_HALF_ULP if stored_bf16 == "both" else (BF16_HALF_ULP if stored_bf16 else 0.0)
    elem = float(np.max(d - q * np.abs(ref))) / rms
    rel_rms = float(np.sqrt(np.mean(d ** 2))) / rms
    return max(rel_rms, elem)


# Every check's figure, for the optional per-test error report (conftest.py).
RECORD: list[tuple[str, str, float, float]] = []


def check(got, ref, mode, what, stored_bf16=None):
    e = err(got, ref, mode, stored_bf16)
    tol = TOL_F32_ABS if mode == "f32" else TOL_BF16_REL
    RECORD.append((what, mode, e, tol))
    assert e <= tol, f"{what}: error {e:.3e} > {tol:.1e} ({'max abs' if mode == 'f32' else 'rms-relative'})"
    return e


def run_chunk(d, chunk, want_state=True, cu=None, workspace=True):
    """kda_chunk_fwd on the GPU copies of d.  workspace=True passes a torch-allocated
    workspace; None / False passes none, so the library draws its scratch from the
    stream-ordered pool (the same kernels either way)."""
    on = to_dev(d)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, ST = kda.kda_chunk_fwd(on["q"], on["k"], on["v"], on["g"], on["beta"], S0=on["S0"],
                                cu_seqlens=on.get("cu_seqlens") if cu is None else cu.cuda(),
                                chunk=chunk, want_state=want_state, workspace=workspace, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"device status {int(status.item()):#x}"
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
