"""The entry points are stream-ordered and never synchronise, so they can be
captured in a CUDA graph and replayed: the prefill with a caller workspace (its
memset and programmatic-dependent launches), with pool scratch (stream-ordered
allocation and release inside the graph), through the static scratch of the
no-alloc entry point (after a first call outside the capture), the decode step,
the recurrent pass and the chunkwise backward, each replayed as called eagerly."""
import pytest
import torch

import kimi_delta_attention_22_b200 as kda
from kimi_delta_attention_22_b200 import inputs


@pytest.mark.gpu
@pytest.mark.parametrize("workspace", [True, None, "noalloc"])
def test_prefill_graph_replay_equals_eager(workspace):
    d = inputs.draw(2, 300, 4, 128, 128, dtype=torch.bfloat16, s0_std=0.02, seed=808, device="cuda")
    args = (d["q"], d["k"], d["v"], d["g"], d["beta"])
    ws = None
    if workspace is True:
        ws = torch.empty(kda.kda_chunk_fwd_workspace_size(d["q"], d["v"], d["g"]), dtype=torch.uint8,
                         device="cuda")
    out = torch.empty_like(d["v"])
    ST = torch.empty(2, 4, 128, 128, dtype=torch.float32, device="cuda")
    def call(**kw):
        if workspace == "noalloc":
            return kda.kda_chunk_fwd_noalloc(*args, S0=d["S0"], **kw)
        return kda.kda_chunk_fwd(*args, S0=d["S0"], workspace=ws, **kw)

    o_ref, s_ref = call()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):   # warm-up on the capture stream
        call(out=out, S_T=ST)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    out.zero_()
    ST.zero_()
    with torch.cuda.graph(g):
        call(out=out, S_T=ST)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, o_ref) and torch.equal(ST, s_ref)


@pytest.mark.gpu
def test_decode_and_recurrent_graph_replay():
    N, H, T = 8, 4, 3
    d = inputs.draw(N, T, H, 128, 128, dtype=torch.bfloat16, s0_std=0.05, seed=809, device="cuda")
    steps = [{n: d[n][:, t].contiguous() for n in ("q", "k", "v", "g", "beta")} for t in range(T)]
    # eager reference: T decode steps, then a recurrent pass over the same tokens
    S_ref = d["S0"].clone()
    outs_ref = [kda.kda_decode_step(st["q"], st["k"], st["v"], st["g"], st["beta"], S_ref) for st in steps]
    S2_ref = S_ref.clone()
    o2_ref = kda.kda_recurrent_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S2_ref)
    torch.cuda.synchronize()

    S = torch.empty_like(d["S0"])
    S2 = torch.empty_like(d["S0"])
    outs = [torch.empty(N, H, 128, dtype=torch.bfloat16, device="cuda") for _ in range(T)]
    o2 = torch.empty_like(d["v"])

    def body():
        S.copy_(d["S0"])
        for st, o in zip(steps, outs):
            kda.kda_decode_step(st["q"], st["k"], st["v"], st["g"], st["beta"], S, out=o)
        S2.copy_(S)
        kda.kda_recurrent_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S2, out=o2)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        body()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        body()
    g.replay()
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(outs, outs_ref))
    assert torch.equal(S, S_ref) and torch.equal(o2, o2_ref) and torch.equal(S2, S2_ref)


@pytest.mark.gpu
@pytest.mark.parametrize("qk_heads", [None, 2])
def test_chunk_bwd_graph_replay_equals_eager(qk_heads):
    """The chunkwise backward with a caller workspace (five launches, the later ones
    programmatic-dependent; grouped heads add a memset of dq, dk) replays in a graph
    as called eagerly: bit-identical, or to fp32 rounding where grouped heads sum dq, dk
    with atomics."""
    import ctypes

    B, T, H = 2, 150, 4
    d = inputs.draw(B, T, H, 128, 128, dtype=torch.bfloat16, s0_std=0.02, seed=809, device="cuda",
                    qk_heads=qk_heads)
    gen = torch.Generator(device="cuda").manual_seed(810)
    d_out = torch.randn(B, T, H, 128, device="cuda", generator=gen).to(torch.bfloat16)
    d_ST = torch.randn(B, H, 128, 128, device="cuda", generator=gen)
    sh = kda.Shape(B, T, H, 128, 128, B, kda.KDA_BF16, kda.KDA_GATE_CHANNEL, 64, None, qk_heads or 0)
    ws = torch.empty(kda.load_library().kda_chunk_bwd_workspace_size(ctypes.byref(sh), 0), dtype=torch.uint8,
                     device="cuda")

    def call():
        return kda.kda_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], d_out, d_ST=d_ST,
                                 workspace=ws)

    ref = call()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        res = call()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    for n in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        if qk_heads and n in ("dq", "dk"):
            assert torch.allclose(res[n], ref[n], rtol=0, atol=1e-6 * float(ref[n].abs().max())), n
        else:
            assert torch.equal(res[n], ref[n]), n
