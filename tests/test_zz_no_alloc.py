"""kda_chunk_fwd_noalloc: the prefill for callers that cannot allocate device
memory (an allocator that owns all of it, a capture region that forbids
allocation nodes, a host that forbids cudaMalloc), run on the library's own
static device scratch.  On the CPU: the symbol is exported and host validation
answers before any device call, including the rejection of shapes too large for
the scratch.  On the GPU: parity with the oracle, and the same bits as the
caller-workspace call, on two calls in a row (the array keeps the previous
call's contents)."""
import ctypes

import pytest
import torch

import kimi_delta_attention_22_b200 as kda
from kimi_delta_attention_22_b200 import build as kbuild
from kimi_delta_attention_22_b200 import inputs
from parity import check, oracle_chunk, sampled_pairs_oracle, to_dev

STATIC_SCRATCH = 160 << 20


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load_library()


def test_noalloc_exported_and_validates(lib):
    assert hasattr(lib, "kda_chunk_fwd_noalloc")
    A = ctypes.c_void_p(0x10000)
    # no shape
    assert lib.kda_chunk_fwd_noalloc(None, A, A, A, A, A, None, None, A, None, None) == 1
    # zero sequences: valid, nothing launched, no device call
    sh = kda.Shape(0, 64, 2, 128, 128, 0, kda.KDA_BF16, kda.KDA_GATE_CHANNEL, 64, None)
    assert lib.kda_chunk_fwd_noalloc(ctypes.byref(sh), A, A, A, A, A, None, None, A, None, None) == 0
    # an unsupported head size is rejected by the same checks as kda_chunk_fwd
    sh = kda.Shape(1, 64, 2, 24, 24, 1, kda.KDA_F32, kda.KDA_GATE_CHANNEL, 16, None)
    assert lib.kda_chunk_fwd_noalloc(ctypes.byref(sh), A, A, A, A, A, None, None, A, None, None) == 2


def test_workspace_sizes_against_the_static_scratch(lib):
    """The bench prefill fits the static scratch; a 4096-token, 48-head one does not."""
    fits = kda.Shape(4, 2048, 16, 128, 128, 4, kda.KDA_BF16, kda.KDA_GATE_CHANNEL, 64, None)
    over = kda.Shape(1, 4096, 48, 128, 128, 1, kda.KDA_BF16, kda.KDA_GATE_CHANNEL, 64, None)
    assert lib.kda_chunk_fwd_workspace_size(ctypes.byref(fits), 0) <= STATIC_SCRATCH
    assert lib.kda_chunk_fwd_workspace_size(ctypes.byref(over), 0) > STATIC_SCRATCH


@pytest.mark.gpu
def test_noalloc_small_matches_oracle():
    d = inputs.draw(2, 200, 3, 128, 128, dtype=torch.bfloat16, s0_std=0.02, seed=2203)
    on = to_dev(d)
    out, ST = kda.kda_chunk_fwd_noalloc(on["q"], on["k"], on["v"], on["g"], on["beta"], S0=on["S0"])
    torch.cuda.synchronize()
    ro, rs = oracle_chunk(d, "channel")
    check(out, ro, "bf16", "out")
    check(ST, rs, "bf16", "S_T")


@pytest.mark.gpu
def test_noalloc_equals_workspace_schedule_full_size():
    w = inputs.WORKLOADS["prefill_b4_h16_t2048"]
    d = inputs.workload_inputs(w, device="cuda")
    args = (d["q"], d["k"], d["v"], d["g"], d["beta"])
    o1, s1 = kda.kda_chunk_fwd_noalloc(*args, S0=d["S0"], chunk=w.chunk)
    o2, s2 = kda.kda_chunk_fwd(*args, S0=d["S0"], chunk=w.chunk, workspace=True)
    torch.cuda.synchronize()
    # the same kernels on the same inputs: bit-identical
    assert torch.equal(o1, o2) and torch.equal(s1, s2)
    cpu = {k: (None if v is None else v.cpu()) for k, v in d.items()}
    for (n, h), (ro, rs) in sampled_pairs_oracle(cpu, [(1, 7)], w.gate_mode).items():
        check(o1[n, :, h], ro, "bf16", f"out ({n},{h})")
        check(s1[n, h], rs, "bf16", f"S_T ({n},{h})")


def test_noalloc_rejects_shapes_over_the_static_scratch(lib):
    """A shape whose scratch exceeds the static array returns KDA_ERR_TOO_LARGE before
    anything is launched (the pointers are never touched, so fake ones do)."""
    A = ctypes.c_void_p(0x10000)
    over = kda.Shape(1, 4096, 48, 128, 128, 1, kda.KDA_BF16, kda.KDA_GATE_CHANNEL, 64, None)
    assert lib.kda_chunk_fwd_noalloc(ctypes.byref(over), A, A, A, A, A, None, None, A, None, None) == 6
    assert "static array" in kda.kda_status_str(6)


@pytest.mark.gpu
def test_noalloc_two_calls_in_a_row_equal_workspace():
    """Two different inputs back to back through the shared array: each call equals the
    caller-workspace call bit for bit (the same kernels), whatever the array held."""
    for seed in (2206, 2207):
        d = inputs.draw(3, 321, 5, 128, 128, dtype=torch.bfloat16, s0_std=0.02, seed=seed)
        on = to_dev(d)
        args = (on["q"], on["k"], on["v"], on["g"], on["beta"])
        o1, s1 = kda.kda_chunk_fwd_noalloc(*args, S0=on["S0"])
        o2, s2 = kda.kda_chunk_fwd(*args, S0=on["S0"], workspace=True)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(s1, s2)
        ro, rs = oracle_chunk(d, "channel")
        check(o1, ro, "bf16", f"out (seed {seed})")
        check(s1, rs, "bf16", f"S_T (seed {seed})")


@pytest.mark.gpu
def test_noalloc_grouped_value_heads_equals_workspace():
    """Grouped value heads through the static scratch: the same kernels and bits as
    the caller-workspace call."""
    d = inputs.draw(2, 200, 8, 128, 128, dtype=torch.bfloat16, s0_std=0.02, seed=2205, qk_heads=2)
    on = to_dev(d)
    args = (on["q"], on["k"], on["v"], on["g"], on["beta"])
    o1, s1 = kda.kda_chunk_fwd_noalloc(*args, S0=on["S0"])
    o2, s2 = kda.kda_chunk_fwd(*args, S0=on["S0"], workspace=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)
