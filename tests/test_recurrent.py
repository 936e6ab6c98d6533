"""kda_recurrent_fwd: the fused recurrent pass over a short run of tokens.

CPU: the symbol is exported and host validation answers before any launch.
GPU: element-wise parity with the float64 oracle (token loop from S0 = S),
bit-for-bit equality with T calls of kda_decode_step (the same per-token
arithmetic), agreement with the chunkwise prefill, and a full-size run at the
decode workload's shape sampled against the oracle."""
import ctypes

import pytest
import torch

import kimi_delta_attention_22_b200 as kda
import oracle
from kimi_delta_attention_22_b200 import build as kbuild
from kimi_delta_attention_22_b200 import inputs
from parity import check, to_dev


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load_library()


def _shape(N=1, T=4, H=2, dk=128, dv=128, dtype=kda.KDA_BF16, gate=kda.KDA_GATE_CHANNEL, num=None):
    return kda.Shape(N, T, H, dk, dv, N if num is None else num, dtype, gate, 0, None)


def test_recurrent_exported_and_validates(lib):
    assert hasattr(lib, "kda_recurrent_fwd")
    A = ctypes.c_void_p(0x10000)

    def call(sh, g=A, S=A, q=A):
        return lib.kda_recurrent_fwd(None if sh is None else ctypes.byref(sh), q, A, A, g, A, S, A, None)

    assert call(None) == 1
    assert call(_shape(N=0)) == 0                                   # nothing to do
    assert call(_shape(N=2, T=0)) == 0                              # zero tokens: S unchanged
    assert call(_shape(N=2, num=3)) == 1                            # num_seqs must equal N
    assert call(_shape(N=0, gate=kda.KDA_GATE_NONE)) == 1           # NONE needs g == NULL
    assert call(_shape(N=0, dk=64)) == 2                            # d_k = 128 only
    assert call(_shape(N=0), S=ctypes.c_void_p(0x10008)) == 3       # S 16-byte aligned
    assert call(_shape(N=2), S=None) == 1


def _draw(N, T, H, dv, dtype, gate, seed):
    d = inputs.draw(N, T, H, 128, dv, dtype=dtype, gate=gate, s0_std=0.05, seed=seed)
    return d


def _oracle(d, gate):
    return oracle.forward(d["q"], d["k"], d["v"], d["g"], d["beta"], S0=d["S0"], gate=gate)


CASES = [
    # N, T, H, d_v, dtype, gate
    (2, 9, 3, 128, torch.bfloat16, "channel"),
    (1, 16, 2, 128, torch.float32, "channel"),
    (3, 5, 2, 96, torch.bfloat16, "scalar"),
    (2, 7, 1, 200, torch.float32, "none"),
    (1, 1, 4, 128, torch.bfloat16, "channel_strong"),
    (2, 40, 2, 128, torch.bfloat16, "channel_extreme"),
]


@pytest.mark.gpu
@pytest.mark.parametrize("N,T,H,dv,dtype,gate", CASES)
def test_recurrent_matches_oracle(N, T, H, dv, dtype, gate):
    d = _draw(N, T, H, dv, dtype, gate, seed=N * 100 + T * 10 + H)
    on = to_dev(d)
    S = on["S0"].clone()
    out = kda.kda_recurrent_fwd(on["q"], on["k"], on["v"], on["g"], on["beta"], S)
    torch.cuda.synchronize()
    gm = "channel" if gate.startswith("channel") else gate
    ro, rs = _oracle(d, gm)
    mode = "f32" if dtype == torch.float32 else "bf16"
    check(out, ro, mode, "out")
    check(S, rs, mode, "S")


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_recurrent_equals_decode_steps(dtype):
    """T tokens in one call == T decode steps: the same per-token arithmetic, bit for bit."""
    N, T, H, dv = 3, 6, 2, 128
    d = to_dev(_draw(N, T, H, dv, dtype, "channel", seed=61))
    S1 = d["S0"].clone()
    o1 = kda.kda_recurrent_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S1)
    S2 = d["S0"].clone()
    o2 = torch.empty_like(o1)
    for t in range(T):
        o2[:, t] = kda.kda_decode_step(d["q"][:, t].contiguous(), d["k"][:, t].contiguous(),
                                       d["v"][:, t].contiguous(), d["g"][:, t].contiguous(),
                                       d["beta"][:, t].contiguous(), S2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


@pytest.mark.gpu
def test_recurrent_agrees_with_chunkwise_prefill():
    d = to_dev(_draw(2, 130, 2, 128, torch.bfloat16, "channel", seed=62))
    S = d["S0"].clone()
    o1 = kda.kda_recurrent_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S)
    o2, s2 = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S0=d["S0"])
    torch.cuda.synchronize()
    check(o1, o2.float().cpu().double(), "bf16", "out vs chunkwise")
    check(S, s2.cpu().double(), "bf16", "S vs chunkwise")


@pytest.mark.gpu
def test_recurrent_full_size_decode_shape():
    """N = 256, H = 32, d = 128 (the decode workload's shape), 16 tokens per call;
    sampled (sequence, head) pairs against the oracle."""
    N, T, H = 256, 16, 32
    d = inputs.draw(N, T, H, 128, 128, dtype=torch.bfloat16, gate="channel", s0_std=0.05, seed=63,
                    device="cuda")
    S = d["S0"].clone()
    out = kda.kda_recurrent_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S)
    torch.cuda.synchronize()
    cpu = {k: (None if v is None else v.cpu()) for k, v in d.items()}
    for n, h in [(0, 0), (255, 31), (97, 13)]:
        sl = lambda t: t[n:n + 1, :, h:h + 1]
        ro, rs = oracle.forward(sl(cpu["q"]), sl(cpu["k"]), sl(cpu["v"]), sl(cpu["g"]), sl(cpu["beta"]),
                                S0=cpu["S0"][n:n + 1, h:h + 1], gate="channel")
        check(out[n, :, h], ro[0, :, 0], "bf16", f"out ({n},{h})")
        check(S[n, h], rs[0, 0], "bf16", f"S ({n},{h})")
