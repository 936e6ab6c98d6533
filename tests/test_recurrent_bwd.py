"""kda_recurrent_bwd: gradients of the token loop.

CPU: host validation answers before any launch.
GPU: every gradient against the float64 autograd reference (oracle/backward.py)
on the same inputs, across gate modes, dtypes, grouped value heads, ragged
segment lengths and value widths that do not fill a row block.

Tolerance: the kernel accumulates in fp32 (with atomics for the cross-row
sums), so each gradient tensor is compared with max |gpu - ref| <= 2e-4 *
max(1, max |ref|)."""
import ctypes

import numpy as np
import pytest
import torch

import kimi_delta_attention_22_b200 as kda
from kimi_delta_attention_22_b200 import build as kbuild
from kimi_delta_attention_22_b200 import inputs
from oracle import backward as ob

TOL = 2e-4


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load_library()


def test_bwd_validation(lib):
    A = ctypes.c_void_p(0x10000)

    def call(sh, g=A, dg=A, ws=A, nbytes=1 << 30, S0=None):
        return lib.kda_recurrent_bwd(ctypes.byref(sh), A, A, A, g, A, S0, A, None, A, A, A, dg, A, None,
                                     ws, nbytes, None)

    sh = kda.Shape(0, 8, 2, 128, 128, 0, kda.KDA_BF16, kda.KDA_GATE_CHANNEL, 0, None, 0)
    assert call(sh) == 0                                                 # N = 0: nothing to do
    assert call(sh, dg=None) == 1                                        # gated needs dg
    sh0 = kda.Shape(0, 8, 2, 128, 128, 0, kda.KDA_BF16, kda.KDA_GATE_NONE, 0, None, 0)
    assert call(sh0, g=None, dg=None) == 0 and call(sh0, g=None) == 1   # no gate: no dg
    assert call(kda.Shape(0, 8, 2, 64, 128, 0, kda.KDA_BF16, kda.KDA_GATE_CHANNEL, 0, None, 0)) == 2
    assert call(sh, S0=ctypes.c_void_p(0x10008)) == 3                   # S0 16-byte aligned
    sh2 = kda.Shape(2, 8, 2, 128, 128, 2, kda.KDA_BF16, kda.KDA_GATE_CHANNEL, 0, None, 0)
    assert call(sh2, nbytes=16) == 1                                     # workspace too small
    assert lib.kda_recurrent_bwd_workspace_size(ctypes.byref(sh2)) == 2 * 2 * 1 * 128 * 128 * 4


def _draw(N, T, H, Hk, dv, dtype, gate, seed):
    d = inputs.draw(N, T, H, 128, dv, dtype=dtype, gate=gate, s0_std=0.1, seed=seed, qk_heads=Hk)
    gen = torch.Generator().manual_seed(seed + 1)
    d["d_out"] = torch.randn(N, T, H, dv, generator=gen).to(dtype)
    d["d_ST"] = torch.randn(N, H, dv, 128, generator=gen)
    return d


def _cmp(got, ref, what):
    got = got.detach().cpu().double().numpy()
    ref = ref.numpy()
    err = float(np.max(np.abs(got - ref))) if got.size else 0.0
    lim = TOL * max(1.0, float(np.max(np.abs(ref))) if ref.size else 1.0)
    assert err <= lim, f"{what}: max abs error {err:.3e} > {lim:.3e}"


CASES = [
    # N, T, H, Hk, d_v, dtype, gate
    (2, 37, 2, 2, 128, torch.float32, "channel"),
    (1, 16, 4, 2, 128, torch.bfloat16, "channel"),
    (2, 5, 3, 1, 40, torch.float32, "scalar"),
    (1, 33, 2, 2, 128, torch.float32, "none"),
    (1, 1, 2, 2, 128, torch.bfloat16, "channel_strong"),
    (4, 13, 40, 20, 128, torch.bfloat16, "channel"),   # 1280 CTAs: the half-window kernel
]


@pytest.mark.gpu
@pytest.mark.parametrize("N,T,H,Hk,dv,dtype,gate", CASES)
def test_bwd_matches_reference(N, T, H, Hk, dv, dtype, gate):
    d = _draw(N, T, H, Hk, dv, dtype, gate, seed=N * 31 + T * 7 + H)
    gm = "channel" if gate.startswith("channel") else gate
    ref = ob.backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], d["d_out"], d["d_ST"], gate=gm)
    on = {n: (None if x is None else x.cuda()) for n, x in d.items()}
    got = kda.kda_recurrent_bwd(on["q"], on["k"], on["v"], on["g"], on["beta"], on["S0"], on["d_out"],
                                on["d_ST"])
    torch.cuda.synchronize()
    for n in ("dq", "dk", "dv", "dbeta", "dS0"):
        _cmp(got[n], ref[n], n)
    if gm == "none":
        assert got["dg"] is None
    else:
        _cmp(got["dg"], ref["dg"], "dg")


@pytest.mark.gpu
def test_bwd_zero_state_and_no_state_gradient():
    """S0 = None (zero state), d_ST = None, dS0 not requested."""
    d = _draw(1, 20, 2, 2, 128, torch.float32, "channel", seed=99)
    ref = ob.backward(d["q"], d["k"], d["v"], d["g"], d["beta"], None, d["d_out"], None, gate="channel")
    on = {n: (None if x is None else x.cuda()) for n, x in d.items()}
    got = kda.kda_recurrent_bwd(on["q"], on["k"], on["v"], on["g"], on["beta"], None, on["d_out"], None,
                                want_dS0=False)
    torch.cuda.synchronize()
    assert got["dS0"] is None
    for n in ("dq", "dk", "dv", "dg", "dbeta"):
        _cmp(got[n], ref[n], n)
