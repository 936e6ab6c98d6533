"""kda_chunk_bwd: gradients of the chunkwise prefill.

CPU: the symbol is exported and host validation answers before any launch.
GPU: every gradient (dq, dk, dv, dg, dbeta, dS0) against the float64 autograd
of the token loop (oracle/backward.py) on the same inputs: the three gate modes,
strong decay, grouped value heads, ragged tails, packed sequences (one of them
empty), no initial state and no final-state gradient, and sampled (sequence,
head) pairs of the 4 x 16 x 2048 prefill.

Tolerance: the bf16 criterion of the forward -- per tensor, the worst
element-wise error relative to the RMS of the oracle's tensor, <= 2e-2 (the
reverse state scan multiplies fp16 operands into fp32 accumulators, as the
forward scan does; everything else is fp32)."""
import ctypes

import numpy as np
import pytest
import torch

import kimi_delta_attention_22_b200 as kda
from kimi_delta_attention_22_b200 import build as kbuild
from kimi_delta_attention_22_b200 import inputs
from oracle import backward as ob
from parity import check

NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dS0")


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load_library()


def test_chunk_bwd_validation(lib):
    A = ctypes.c_void_p(0x10000)

    def call(sh, g=A, dg=A, ws=None, nbytes=0, cu=None, q=A, dS0=None):
        return lib.kda_chunk_bwd(ctypes.byref(sh), q, A, A, g, A, None, cu, A, None, A, A, A, dg, A, dS0,
                                 ws, nbytes, None)

    def shape(B=2, T=64, H=2, d=128, n=None, dtype=kda.KDA_BF16, gate=kda.KDA_GATE_CHANNEL, chunk=64, Hk=0):
        return kda.Shape(B, T, H, d, d, B if n is None else n, dtype, gate, chunk, None, Hk)

    assert call(shape(B=0, n=0)) == 0                                   # no sequences: nothing to do
    assert call(shape(), dg=None) == 1                                  # a gate needs dg
    assert call(shape(gate=kda.KDA_GATE_NONE), g=None) == 1             # no gate: no dg
    assert call(shape(gate=kda.KDA_GATE_NONE), g=None, dg=None) != 1
    assert call(shape(dtype=kda.KDA_F32)) == 2                          # bf16 only
    assert call(shape(d=64)) == 2                                       # d_k = d_v = 128
    assert call(shape(chunk=32)) == 2                                   # chunk 64
    assert call(shape(Hk=3)) == 1                                       # Hk must divide H
    assert call(shape(), q=ctypes.c_void_p(0x10008)) == 3               # q 16-byte aligned
    assert call(shape(), dS0=ctypes.c_void_p(0x10004)) == 3             # dS0 16-byte aligned
    assert call(shape(), ws=ctypes.c_void_p(0x10080), nbytes=1 << 40) == 3   # workspace 256-byte aligned
    assert call(shape(), ws=A, nbytes=16) == 1                          # workspace too small
    assert call(shape(B=2, n=3)) == 1                                   # dense: num_seqs == B
    assert call(shape(B=2, n=2), cu=A) == 1                             # packed: B == 1


def test_chunk_bwd_workspace_size(lib):
    sh = kda.Shape(4, 2048, 16, 128, 128, 4, kda.KDA_BF16, kda.KDA_GATE_CHANNEL, 64, None, 0)
    units = 4 * 32 * 16
    per = 74240 + 2 * 65536 + 32768 + 3 * 16384 + 16384
    nbytes = lib.kda_chunk_bwd_workspace_size(ctypes.byref(sh), 0)
    # plus the forward's header: the slow-chunk list (one int32 per unit, and a count)
    assert units * per <= nbytes <= units * per + 4 * (units + 1) + 1024
    assert nbytes > lib.kda_chunk_fwd_workspace_size(ctypes.byref(sh), 0)
    bad = kda.Shape(4, 2048, 16, 64, 64, 4, kda.KDA_BF16, kda.KDA_GATE_CHANNEL, 64, None, 0)
    assert lib.kda_chunk_bwd_workspace_size(ctypes.byref(bad), 0) == 0


def _draw(B, T, H, gate, seed, Hk=None, s0=0.1, dst=True, beta="sigmoid"):
    d = inputs.draw(B, T, H, 128, 128, dtype=torch.bfloat16, gate=gate, beta=beta, s0_std=s0, seed=seed,
                    qk_heads=Hk)
    gen = torch.Generator().manual_seed(seed + 1)
    d["d_out"] = torch.randn(B, T, H, 128, generator=gen).to(torch.bfloat16)
    d["d_ST"] = torch.randn(B, H, 128, 128, generator=gen) if dst else None
    return d


def _mode(gate):
    return "channel" if gate.startswith("channel") else gate


def _gpu(d, cu=None, **kw):
    on = {k: (None if v is None else v.cuda()) for k, v in d.items()}
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = kda.kda_chunk_bwd(on["q"], on["k"], on["v"], on["g"], on["beta"], on["S0"], on["d_out"],
                            d_ST=on["d_ST"], cu_seqlens=None if cu is None else cu.cuda(), dev_status=status, **kw)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"device status {int(status.item()):#x}"
    return res


def _compare(got, ref, what):
    for n in NAMES:
        if ref[n] is None:
            continue
        assert got[n] is not None, f"{what}: {n} missing"
        check(got[n], ref[n].numpy(), "bf16", f"{what} {n}", stored_bf16=False)


@pytest.mark.gpu
@pytest.mark.parametrize("gate", ["channel", "scalar", "none", "channel_strong", "channel_extreme"])
def test_chunk_bwd_dense_matches_autograd(gate):
    d = _draw(2, 150, 2, gate, seed=3100 + len(gate))
    got = _gpu(d)
    ref = ob.backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], d["d_out"], d["d_ST"], gate=_mode(gate))
    _compare(got, ref, gate)


@pytest.mark.gpu
def test_chunk_bwd_mixed_decay_regimes():
    """Chunks of one call needing one decay reference, two and sub-block references
    (the gate of test_parity_gpu.mixed_decay_gate), ragged tail."""
    from test_parity_gpu import mixed_decay_gate

    d = _draw(2, 300, 2, "channel", seed=3130)
    d["g"] = mixed_decay_gate(2, 300, 2, seed=3131)
    got = _gpu(d)
    ref = ob.backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], d["d_out"], d["d_ST"], gate="channel")
    _compare(got, ref, "mixed")


@pytest.mark.gpu
@pytest.mark.parametrize("gate", ["channel_extreme", "mixed"])
def test_chunk_bwd_independent_of_scratch_contents(gate):
    """The gradients do not depend on what the workspace held before the call: a
    workspace of zero bytes and one of 0xFF bytes (NaN in every float format) give the
    same, finite results."""
    if gate == "mixed":
        from test_parity_gpu import mixed_decay_gate

        d = _draw(2, 300, 2, "channel", seed=3140)
        d["g"] = mixed_decay_gate(2, 300, 2, seed=3141)
    else:
        d = _draw(2, 150, 2, gate, seed=3142)
    sh = kda.Shape(2, d["v"].shape[1], 2, 128, 128, 2, kda.KDA_BF16, kda.KDA_GATE_CHANNEL, 64, None, 0)
    nbytes = kda.load_library().kda_chunk_bwd_workspace_size(ctypes.byref(sh), 0)
    res = [_gpu(d, workspace=torch.full((nbytes,), fill, dtype=torch.uint8, device="cuda")) for fill in (0, 255)]
    for n in NAMES:
        assert torch.isfinite(res[0][n]).all(), n
        assert torch.equal(res[0][n], res[1][n]), n


@pytest.mark.gpu
def test_chunk_bwd_grouped_heads_no_state():
    """4 value heads over 2 query/key heads (dq, dk summed over the group), zero
    initial state, no final-state gradient, beta = 1."""
    d = _draw(1, 200, 4, "channel", seed=3111, Hk=2, s0=None, dst=False, beta="one")
    got = _gpu(d, want_dS0=False)
    ref = ob.backward(d["q"], d["k"], d["v"], d["g"], d["beta"], None, d["d_out"], None, gate="channel")
    _compare(got, ref, "grouped")


@pytest.mark.gpu
def test_chunk_bwd_varlen_matches_per_sequence_autograd():
    """Packed sequences of 37, 0, 163, 64 and 69 tokens (ragged tails, an empty one, an
    exact chunk): each against the token loop of its own slice and state."""
    lens = [37, 0, 163, 64, 69]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    T = int(cu[-1])
    d = _draw(1, T, 2, "channel", seed=3120)
    d["S0"] = 0.1 * torch.randn(len(lens), 2, 128, 128, generator=torch.Generator().manual_seed(3121))
    d["d_ST"] = torch.randn(len(lens), 2, 128, 128, generator=torch.Generator().manual_seed(3122))
    got = _gpu(d, cu=cu)
    for n, (a, b) in enumerate(zip(cu[:-1].tolist(), cu[1:].tolist())):
        sl = slice(a, b)
        if b == a:   # empty sequence: dS0 = d_ST
            check(got["dS0"][n], d["d_ST"][n].numpy(), "bf16", f"seq {n} dS0", stored_bf16=False)
            continue
        ref = ob.backward(d["q"][:, sl], d["k"][:, sl], d["v"][:, sl], d["g"][:, sl], d["beta"][:, sl],
                          d["S0"][n:n + 1], d["d_out"][:, sl], d["d_ST"][n:n + 1], gate="channel")
        part = {k: (None if got[k] is None else got[k][:, sl]) for k in NAMES if k != "dS0"}
        part["dS0"] = got["dS0"][n:n + 1]
        _compare(part, ref, f"seq {n}")


@pytest.mark.gpu
def test_chunk_bwd_pool_equals_workspace_and_is_deterministic():
    d = _draw(2, 300, 3, "channel", seed=3130)
    r1 = _gpu(d, workspace=True)
    r2 = _gpu(d, workspace=None)
    r3 = _gpu(d, workspace=True)
    for n in NAMES:
        assert torch.equal(r1[n], r2[n]) and torch.equal(r1[n], r3[n]), n


@pytest.mark.gpu
def test_chunk_bwd_no_tokens():
    """T = 0: the state passes through, so dS0 = d_ST."""
    d = _draw(2, 0, 2, "channel", seed=3140)
    got = _gpu(d)
    assert torch.equal(got["dS0"].cpu(), d["d_ST"])


@pytest.mark.gpu
@pytest.mark.parametrize("pair", [(1, 7), (3, 0)])
def test_chunk_bwd_full_size_sampled_pairs(pair):
    """The 4 x 16 x 2048 prefill in one call; the sampled (sequence, head) pair's
    gradients against autograd of its own token loop."""
    w = inputs.WORKLOADS["prefill_b4_h16_t2048"]
    d = inputs.workload_inputs(w)
    gen = torch.Generator().manual_seed(3150)
    d["d_out"] = torch.randn(w.B, w.T, w.H, 128, generator=gen).to(torch.bfloat16)
    d["d_ST"] = torch.randn(w.B, w.H, 128, 128, generator=gen)
    got = _gpu(d)
    n, h = pair
    one = {k: d[k][n:n + 1, :, h:h + 1] for k in ("q", "k", "v", "g", "d_out")}
    ref = ob.backward(one["q"], one["k"], one["v"], one["g"], d["beta"][n:n + 1, :, h:h + 1],
                      d["S0"][n:n + 1, h:h + 1], one["d_out"], d["d_ST"][n:n + 1, h:h + 1], gate="channel")
    part = {k: got[k][n:n + 1, :, h:h + 1] for k in ("dq", "dk", "dv", "dg", "dbeta")}
    part["dS0"] = got["dS0"][n:n + 1, h:h + 1]
    _compare(part, ref, f"pair {pair}")
