"""Grouped value heads: H value heads (v, g, beta, state, out) share Hk < H
query/key heads, value head h reading q/k head h // (H // Hk).

CPU: host validation (q/k heads must divide H) answers before any launch.
GPU: every entry point against the float64 oracle, and bit-for-bit against the
same call with each q/k head repeated for its value heads (the kernels read the
same values either way, so the results must be the same bits)."""
import ctypes

import pytest
import torch

import kimi_delta_attention_22_b200 as kda
import oracle
from kimi_delta_attention_22_b200 import build as kbuild
from kimi_delta_attention_22_b200 import inputs
from parity import check, oracle_chunk, run_chunk, sampled_pairs_oracle, to_dev


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load_library()


def test_qk_heads_must_divide_value_heads(lib):
    A = ctypes.c_void_p(0x10000)
    for hk, want in [(0, 0), (6, 0), (3, 0), (2, 0), (1, 0), (4, 1), (7, 1), (-2, 1)]:
        # N = 0: validation only, nothing launched
        sh = kda.Shape(0, 1, 6, 128, 128, 0, kda.KDA_BF16, kda.KDA_GATE_CHANNEL, 64, None, hk)
        assert lib.kda_decode_step(ctypes.byref(sh), A, A, A, A, A, A, A, None) == want, hk
        assert lib.kda_recurrent_fwd(ctypes.byref(sh), A, A, A, A, A, A, A, None) == want, hk
        sh2 = kda.Shape(0, 64, 6, 128, 128, 0, kda.KDA_BF16, kda.KDA_GATE_CHANNEL, 64, None, hk)
        st = lib.kda_chunk_fwd(ctypes.byref(sh2), A, A, A, A, A, None, None, A, None, None, 0, None)
        assert st == want, hk


def _rep(d, G):
    """The same inputs with each q/k head repeated for its G value heads."""
    e = dict(d)
    e["q"] = d["q"].repeat_interleave(G, dim=-2).contiguous()
    e["k"] = d["k"].repeat_interleave(G, dim=-2).contiguous()
    return e


CHUNK_CASES = [
    # B, T, H, Hk, dtype, gate, chunk
    (2, 130, 4, 2, torch.bfloat16, "channel", 64),
    (1, 200, 6, 2, torch.bfloat16, "scalar", 64),
    (2, 97, 4, 1, torch.bfloat16, "channel_strong", 64),
    (2, 70, 3, 1, torch.float32, "channel", 32),
]


@pytest.mark.gpu
@pytest.mark.parametrize("B,T,H,Hk,dtype,gate,chunk", CHUNK_CASES)
def test_chunk_grouped_matches_oracle_and_repeated(B, T, H, Hk, dtype, gate, chunk):
    dk = dv = 128 if dtype == torch.bfloat16 else 64
    d = inputs.draw(B, T, H, dk, dv, dtype=dtype, gate=gate, s0_std=0.02, seed=B * 100 + T + H * 7 + Hk,
                    qk_heads=Hk)
    gm = "channel" if gate.startswith("channel") else gate
    ro, rs = oracle_chunk(d, gm)
    mode = "f32" if dtype == torch.float32 else "bf16"
    scheds = [True, None] if dtype == torch.bfloat16 else [True]
    for ws in scheds:
        out, ST = run_chunk(d, chunk, workspace=ws)
        check(out, ro, mode, f"out (workspace={ws})")
        check(ST, rs, mode, f"S_T (workspace={ws})")
        o2, s2 = run_chunk(_rep(d, H // Hk), chunk, workspace=ws)
        assert torch.equal(out, o2) and torch.equal(ST, s2), f"grouped != repeated (workspace={ws})"


@pytest.mark.gpu
def test_varlen_grouped():
    lens = [1, 64, 130, 0, 77]
    cu = torch.tensor([0] + list(torch.cumsum(torch.tensor(lens), 0).tolist()), dtype=torch.int32)
    d = inputs.draw(1, int(cu[-1]), 4, 128, 128, dtype=torch.bfloat16, s0_std=0.02, num_states=len(lens),
                    seed=515, qk_heads=2)
    d["cu_seqlens"] = cu
    ro, rs = oracle_chunk(d, "channel")
    for ws in (True, None):
        out, ST = run_chunk(d, 64, workspace=ws)
        check(out, ro, "bf16", "out")
        check(ST, rs, "bf16", "S_T")


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_and_recurrent_grouped(dtype):
    N, T, H, Hk = 3, 5, 4, 2
    d = to_dev(inputs.draw(N, T, H, 128, 128, dtype=dtype, s0_std=0.05, seed=616, qk_heads=Hk))
    cpu = {k: (None if v is None else v.cpu()) for k, v in d.items()}
    ro, rs = oracle.forward(cpu["q"], cpu["k"], cpu["v"], cpu["g"], cpu["beta"], S0=cpu["S0"], gate="channel")
    mode = "f32" if dtype == torch.float32 else "bf16"
    S = d["S0"].clone()
    out = kda.kda_recurrent_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S)
    S2 = d["S0"].clone()
    dec = torch.empty_like(out)
    for t in range(T):
        dec[:, t] = kda.kda_decode_step(*(d[n][:, t].contiguous() for n in ("q", "k", "v", "g", "beta")), S2)
    e = _rep(d, H // Hk)
    S3 = d["S0"].clone()
    out3 = kda.kda_recurrent_fwd(e["q"], e["k"], e["v"], e["g"], e["beta"], S3)
    torch.cuda.synchronize()
    check(out, ro, mode, "recurrent out")
    check(S, rs, mode, "recurrent S")
    assert torch.equal(out, dec) and torch.equal(S, S2), "recurrent != decode steps"
    assert torch.equal(out, out3) and torch.equal(S, S3), "grouped != repeated"


@pytest.mark.gpu
def test_grouped_full_size_prefill():
    """B4 H16 T2048 with 4 query/key heads (4 value heads each), both schedules;
    sampled (sequence, value head) pairs against the oracle."""
    d = inputs.draw(4, 2048, 16, 128, 128, dtype=torch.bfloat16, s0_std=0.02, seed=717, qk_heads=4,
                    device="cuda")
    cpu = {k: (None if v is None else v.cpu()) for k, v in d.items()}
    ref = None
    for ws in (True, None):
        out, ST = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S0=d["S0"], workspace=ws)
        torch.cuda.synchronize()
        for (n, h) in [(0, 0), (1, 5), (3, 15), (2, 10)]:
            hk = h // 4
            sl = lambda t, hh: t[n:n + 1, :, hh:hh + 1]
            key = (n, h)
            if ref is None or key not in ref:
                ref = ref or {}
                ro, rs = oracle.forward(sl(cpu["q"], hk), sl(cpu["k"], hk), sl(cpu["v"], h), sl(cpu["g"], h),
                                        sl(cpu["beta"], h), S0=cpu["S0"][n:n + 1, h:h + 1], gate="channel")
                ref[key] = (ro[0, :, 0], rs[0, 0])
            check(out[n, :, h], ref[key][0], "bf16", f"out ({n},{h}) ws={ws}")
            check(ST[n, h], ref[key][1], "bf16", f"S_T ({n},{h}) ws={ws}")
