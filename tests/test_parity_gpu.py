"""GPU parity: the CUDA path through the C ABI against the float64 oracle on
the same seeded inputs (element by element), plus equivalences that hold at
any size.  Tolerances: fp32 mode max |gpu - oracle| <= 1e-4; bf16 mode, per
tensor (outputs and states), max |gpu - oracle| / rms(oracle) <= 2e-2 element by
element, with half a bf16 ulp of the oracle's value allowed on bf16-stored
outputs for the rounding of the stored result (tests/parity.py)."""
import numpy as np
import pytest
import torch

import kimi_delta_attention_22_b200 as kda
import oracle
from kimi_delta_attention_22_b200 import inputs
from parity import (check, err, gate_of, oracle_chunk, run_chunk, sampled_pairs_oracle,
                    sampled_varlen_oracle, to_dev)

pytestmark = pytest.mark.gpu


# ----------------------------------------------------------------- small cases

def test_small_f32_workload():
    """fp32, B=1, H=1, T=64, d=16, chunk 16, zero initial state."""
    d = inputs.workload_inputs("small_f32_t64_d16")
    out, ST = run_chunk(d, 16)
    ro, rs = oracle_chunk(d, "channel")
    check(out, ro, "f32", "out")
    check(ST, rs, "f32", "S_T")


F32_CASES = [
    # dk, dv, chunk, B, T, H, gate, s0
    (16, 32, 16, 2, 100, 2, "channel", True),
    (64, 64, 32, 1, 130, 3, "scalar", False),
    (128, 128, 64, 2, 200, 2, "channel", True),
    (32, 16, 64, 3, 65, 1, "none", True),
    (128, 64, 16, 1, 33, 2, "channel_strong", True),
    (48, 80, 32, 1, 1, 2, "channel", True),
    (128, 128, 64, 1, 150, 2, "channel_extreme", True),
]


@pytest.mark.parametrize("dk,dv,chunk,B,T,H,gate,s0", F32_CASES)
def test_f32_path(dk, dv, chunk, B, T, H, gate, s0):
    d = inputs.draw(B, T, H, dk, dv, dtype=torch.float32, gate=gate, s0_std=0.5 if s0 else None,
                    seed=dk + dv + T)
    out, ST = run_chunk(d, chunk)
    ro, rs = oracle_chunk(d, gate_of(d))
    check(out, ro, "f32", "out")
    check(ST, rs, "f32", "S_T")


BF16_CASES = [
    # B, T, H, gate, beta, s0, chunk
    (2, 200, 3, "channel", "sigmoid", True, 64),
    (1, 64, 2, "channel", "one", False, 64),
    (3, 65, 2, "scalar", "sigmoid", True, 64),
    (2, 130, 2, "none", "one", True, 64),
    (2, 190, 2, "channel_strong", "sigmoid", False, 64),
    (1, 1, 4, "channel", "sigmoid", True, 64),
    (2, 97, 2, "channel", "sigmoid", True, 32),
    (2, 150, 2, "channel_extreme", "sigmoid", True, 64),
    (1, 100, 2, "channel_extreme", "one", True, 32),
]


@pytest.mark.parametrize("schedule", ["workspace", "pool"])
@pytest.mark.parametrize("B,T,H,gate,beta,s0,chunk", BF16_CASES)
def test_bf16(B, T, H, gate, beta, s0, chunk, schedule):
    d = inputs.draw(B, T, H, 128, 128, dtype=torch.bfloat16, gate=gate, beta=beta,
                    s0_std=0.02 if s0 else None, seed=B * 1000 + T + H)
    out, ST = run_chunk(d, chunk, workspace=schedule == "workspace")
    ro, rs = oracle_chunk(d, gate_of(d))
    check(out, ro, "bf16", "out")
    check(ST, rs, "bf16", "S_T")


@pytest.mark.parametrize("gate,qk_div", [("channel", 1), ("channel_strong", 1), ("channel_extreme", 1), ("channel", 2)])
def test_whole_width_scan_matches_oracle(gate, qk_div):
    """More (sequence, head) pairs than SMs take the whole-width (N = 128) state
    scan: 2 x 90 heads, ragged 130-token sequences, one- and sub-block-reference
    chunks, and grouped value heads (two per q/k head); every pair against the oracle."""
    props = torch.cuda.get_device_properties(0)
    B, T, H = 2, 130, max(90, props.multi_processor_count // 2 + 1)
    H += H % 2
    d = inputs.draw(B, T, H, 128, 128, dtype=torch.bfloat16, gate=gate, s0_std=0.02, seed=4242,
                    qk_heads=H // qk_div)
    out, ST = run_chunk(d, 64)
    ro, rs = oracle_chunk(d, "channel")
    check(out, ro, "bf16", "out")
    check(ST, rs, "bf16", "S_T")


def mixed_decay_gate(B, T, H, seed):
    """Per-channel gates whose strength changes from chunk to chunk (64 tokens each):
    -softplus(N(0,1)), -U(0,5), -U(0,10), -U(0,0.2), repeating; the tensor-core path
    takes one decay reference, two references and sub-block references for them."""
    gen = torch.Generator().manual_seed(seed)
    g = torch.empty(B, T, H, 128)
    for c0 in range(0, T, 64):
        n = min(64, T - c0)
        kind = (c0 // 64) % 4
        if kind == 0:
            g[:, c0:c0 + n] = -torch.nn.functional.softplus(torch.randn(B, n, H, 128, generator=gen))
        else:
            g[:, c0:c0 + n] = -(5.0, 10.0, 0.2)[kind - 1] * torch.rand(B, n, H, 128, generator=gen)
    return g


@pytest.mark.parametrize("schedule", ["workspace", "pool"])
def test_mixed_decay_regimes_in_one_call(schedule):
    """One call whose chunks need one reference, two references and sub-block
    references (ragged tail included), against the oracle."""
    d = inputs.draw(2, 300, 2, 128, 128, dtype=torch.bfloat16, s0_std=0.02, seed=91)
    d["g"] = mixed_decay_gate(2, 300, 2, seed=92)
    out, ST = run_chunk(d, 64, workspace=schedule == "workspace")
    ro, rs = oracle_chunk(d, "channel")
    check(out, ro, "bf16", "out")
    check(ST, rs, "bf16", "S_T")


def test_forward_independent_of_scratch_contents():
    """out and S_T do not depend on what the workspace held: zero bytes and 0xFF bytes
    (NaN in every float format) give the same, finite results (all three decay regimes)."""
    import ctypes

    d = inputs.draw(2, 300, 2, 128, 128, dtype=torch.bfloat16, s0_std=0.02, seed=93)
    d["g"] = mixed_decay_gate(2, 300, 2, seed=94)
    sh = kda.Shape(2, 300, 2, 128, 128, 2, kda.KDA_BF16, kda.KDA_GATE_CHANNEL, 64, None, 0)
    nbytes = kda.load_library().kda_chunk_fwd_workspace_size(ctypes.byref(sh), 0)
    res = [run_chunk(d, 64, workspace=torch.full((nbytes,), fill, dtype=torch.uint8, device="cuda"))
           for fill in (0, 255)]
    for a, b in zip(res[0], res[1]):
        assert torch.isfinite(a.float()).all()
        assert torch.equal(a, b)


@pytest.mark.parametrize("schedule", ["workspace", "pool"])
def test_varlen_small_ragged_and_empty(schedule):
    """Packed sequences of lengths 0, 1, 64, 65, 127, 200 (state restarts per
    sequence; the empty one returns S0)."""
    lens = [0, 1, 64, 65, 127, 200]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    d = inputs.draw(1, int(cu[-1]), 2, 128, 128, dtype=torch.bfloat16, s0_std=0.02,
                    num_states=len(lens), seed=77)
    d["cu_seqlens"] = cu
    out, ST = run_chunk(d, 64, workspace=schedule == "workspace")
    ro, rs = oracle_chunk(d, "channel")
    check(out, ro, "bf16", "out")
    check(ST, rs, "bf16", "S_T")
    assert torch.equal(ST[0].cpu(), d["S0"][0]), "empty sequence must return S0 unchanged"


def test_state_optional():
    d = inputs.draw(1, 70, 2, 128, 128, dtype=torch.bfloat16, seed=5)
    out, ST = run_chunk(d, 64, want_state=False)
    assert ST is None
    ro, _ = oracle_chunk(d, "channel")
    check(out, ro, "bf16", "out")


def test_resume_equals_one_pass():
    """chunk_fwd over T1 + T2 tokens == chunk_fwd over T2 resumed from S_T of T1."""
    d = inputs.draw(2, 300, 2, 128, 128, dtype=torch.bfloat16, s0_std=0.02, seed=9)
    on = to_dev(d)
    o_all, s_all = kda.kda_chunk_fwd(on["q"], on["k"], on["v"], on["g"], on["beta"], S0=on["S0"])
    cut = 128
    sl = lambda t, a, b: t[:, a:b].contiguous()
    o1, s1 = kda.kda_chunk_fwd(*(sl(on[n], 0, cut) for n in ("q", "k", "v", "g", "beta")),
                               S0=on["S0"])
    o2, s2 = kda.kda_chunk_fwd(*(sl(on[n], cut, 300) for n in ("q", "k", "v", "g", "beta")),
                               S0=s1)
    torch.cuda.synchronize()
    ro, rs = oracle_chunk(d, "channel")
    check(torch.cat([o1, o2], 1), ro, "bf16", "resumed out")
    check(s2, rs, "bf16", "resumed S_T")
    check(o_all, ro, "bf16", "one-pass out")


def test_chunk_size_invariance_f32():
    d = inputs.draw(2, 150, 2, 64, 64, dtype=torch.float32, s0_std=0.5, seed=31)
    res = [run_chunk(d, c) for c in (16, 32, 64)]
    for o, s in res[1:]:
        assert float((o - res[0][0]).abs().max()) <= 1e-4
        assert float((s - res[0][1]).abs().max()) <= 1e-4


def test_varlen_equals_separate_calls():
    lens = [70, 5, 128]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    d = inputs.draw(1, sum(lens), 2, 128, 128, dtype=torch.bfloat16, s0_std=0.02,
                    num_states=3, seed=41)
    on = to_dev(d)
    ov, sv = kda.kda_chunk_fwd(on["q"], on["k"], on["v"], on["g"], on["beta"], S0=on["S0"],
                               cu_seqlens=cu.cuda())
    for n in range(3):
        a, b = int(cu[n]), int(cu[n + 1])
        sl = lambda t: t[:, a:b].contiguous()
        on_, sn = kda.kda_chunk_fwd(*(sl(on[x]) for x in ("q", "k", "v", "g", "beta")),
                                    S0=on["S0"][n:n + 1].contiguous())
        torch.cuda.synchronize()
        check(on_, ov[:, a:b].double().cpu().numpy(), "bf16", f"varlen vs separate out {n}",
              stored_bf16="both")
        check(sn[0], sv[n].double().cpu().numpy(), "bf16", f"varlen vs separate S_T {n}")


def test_bad_cu_seqlens_sets_device_status():
    """A decreasing cu_seqlens is caught by the kernel's own bounds check: the
    bad sequence is skipped and dev_status records it; nothing faults."""
    cu = torch.tensor([0, 40, 20, 60], dtype=torch.int32, device="cuda")
    d = to_dev(inputs.draw(1, 60, 2, 128, 128, dtype=torch.bfloat16, num_states=3, seed=3))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], cu_seqlens=cu,
                      dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & kda.KDA_DEV_BAD_SEQLENS


def test_decode_small_parity():
    N, H = 3, 2
    S = 0.3 * torch.randn(N, H, 96, 128, generator=torch.Generator().manual_seed(1))  # d_v=96
    for gate in ("channel", "scalar", "none"):
        for dt in (torch.bfloat16, torch.float32):
            d = inputs.draw(1, N, H, 128, 96, dtype=dt, gate=gate, seed=11)
            q, k, v, g, b = (None if d[n] is None else d[n][0] for n in ("q", "k", "v", "g", "beta"))
            Sd = S.clone().cuda()
            o = kda.kda_decode_step(q.cuda(), k.cuda(), v.cuda(), None if g is None else g.cuda(),
                                    b.cuda(), Sd)
            torch.cuda.synchronize()
            ro, rs = oracle.decode_step(q, k, v, g, b, S, gate=gate)
            mode = "f32" if dt == torch.float32 else "bf16"
            check(o, ro, mode, f"decode out {gate} {dt}")
            check(Sd, rs, mode, f"decode S {gate} {dt}")


def test_decode_steps_equal_prefill():
    """T single-token decode steps give the outputs and state of one chunked
    prefill over the same T tokens."""
    B, T, H = 2, 40, 2
    d = to_dev(inputs.draw(B, T, H, 128, 128, dtype=torch.bfloat16, s0_std=0.02, seed=21))
    o_ref, s_ref = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S0=d["S0"])
    S = d["S0"].clone()
    outs = []
    for t in range(T):
        outs.append(kda.kda_decode_step(*(d[n][:, t].contiguous() for n in ("q", "k", "v", "g", "beta")), S))
    torch.cuda.synchronize()
    o_dec = torch.stack(outs, 1)
    check(o_dec, o_ref.double().cpu().numpy(), "bf16", "decode vs prefill out", stored_bf16="both")
    check(S, s_ref.double().cpu().numpy(), "bf16", "decode vs prefill state")


# ------------------------------------------------------- full-size workloads

def _full_dense(name, pairs):
    w = inputs.WORKLOADS[name]
    d = inputs.workload_inputs(w, device="cuda")
    out, ST = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S0=d["S0"],
                                chunk=w.chunk)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(out.float()).all()) and bool(torch.isfinite(ST).all())
    cpu = {k: (None if v is None else v.cpu()) for k, v in d.items()}
    ref = sampled_pairs_oracle(cpu, pairs, w.gate_mode)
    for (n, h), (ro, rs) in ref.items():
        check(out[n, :, h], ro, "bf16", f"{name} out ({n},{h})")
        check(ST[n, h], rs, "bf16", f"{name} S_T ({n},{h})")


def test_prefill_full_size():
    _full_dense("prefill_b4_h16_t2048", [(0, 0), (1, 5), (2, 10), (3, 15)])


@pytest.mark.parametrize("name", [n for n in inputs.WORKLOADS if n.startswith("sweep_")])
def test_sweep_full_size(name):
    _full_dense(name, [(0, 0), (7, 63), (3, 21)])


def test_varlen_full_size():
    w = inputs.WORKLOADS["varlen_h32_t65536"]
    d = inputs.workload_inputs(w, device="cuda")
    out, ST = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S0=None,
                                cu_seqlens=d["cu_seqlens"], chunk=w.chunk)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(out.float()).all())
    cpu = {k: (None if v is None else v.cpu()) for k, v in d.items()}
    pairs = [(0, 0), (7, 31), (3, 17)]
    ref = sampled_varlen_oracle(cpu, pairs, "channel")
    cu = cpu["cu_seqlens"].numpy()
    for (n, h), (ro, rs) in ref.items():
        check(out[0, cu[n]:cu[n + 1], h], ro, "bf16", f"varlen out ({n},{h})")
        check(ST[n, h], rs, "bf16", f"varlen S_T ({n},{h})")


def test_decode_full_size():
    """256 x 32 heads, state from a 512-token prefill, 128 one-token steps.
    The oracle starts from the GPU's post-prefill state (exact fp32) on sampled
    (n, h) pairs and is compared at every step and on the final state; the
    prefill itself is checked on the same pairs."""
    D = inputs.DECODE
    N, H, steps = D["N"], D["H"], D["steps"]
    pre = inputs.draw(N, D["prefill_T"], H, 128, 128, seed=D["seed"], device="cuda")
    _, S = kda.kda_chunk_fwd(pre["q"], pre["k"], pre["v"], pre["g"], pre["beta"])
    torch.cuda.synchronize()
    pairs = [(0, 0), (255, 31), (100, 7)]
    cpu_pre = {k: (None if v is None else v.cpu()) for k, v in pre.items()}
    ref_pre = sampled_pairs_oracle(cpu_pre, pairs, "channel")
    for (n, h), (_, rs) in ref_pre.items():
        check(S[n, h], rs, "bf16", f"decode prefill S ({n},{h})")
    S0 = S.clone()
    dec = inputs.decode_inputs(N, H, 128, 128, steps, D["seed"] + 1000, device="cuda")
    outs = torch.empty(steps, N, H, 128, dtype=torch.bfloat16, device="cuda")
    for t in range(steps):
        kda.kda_decode_step(dec["q"][t], dec["k"][t], dec["v"][t], dec["g"][t], dec["beta"][t], S,
                            out=outs[t])
    torch.cuda.synchronize()
    for n, h in pairs:
        sl = lambda x: x[:, n, h].cpu()[None, :, None]
        ro, rs = oracle.forward(sl(dec["q"]), sl(dec["k"]), sl(dec["v"]), sl(dec["g"]),
                                sl(dec["beta"]), S0=S0[n, h].cpu()[None, None])
        check(outs[:, n, h], ro[0, :, 0], "bf16", f"decode outs ({n},{h})")
        check(S[n, h], rs[0, 0], "bf16", f"decode final S ({n},{h})")
