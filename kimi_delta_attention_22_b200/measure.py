"""Time kda_chunk_fwd on the named synthetic workloads (one GPU).

    python -m kimi_delta_attention_22_b200.measure [--workloads a,b,...] [--schedule workspace|pool]
                                                   [--iters 10] [--warmup 3] [--shape B,T,H]
    python -m kimi_delta_attention_22_b200.measure --recurrent [--tokens 1,4,16,64]
    python -m kimi_delta_attention_22_b200.measure --chunk-backward workload[,workload...]

For each workload: inputs drawn once on the device (kimi_delta_attention_22_b200.inputs),
the prefill's workspace allocated once (--schedule pool: none, so each call takes its
scratch from the stream-ordered pool), `warmup` untimed calls, then `iters`
calls timed one by one with CUDA events on the current stream; the median is reported
with tokens/s, the algorithmic HBM bytes and FLOPs of kimi_delta_attention_22_b200.roofline
and their fractions of MEASURED_PEAKS.json (repository root) when that file exists.
Inputs of the prefill and sweep workloads exceed the 126 MB L2, so consecutive calls do
not re-read them from L2; the small fp32 case is listed for completeness only.
One JSON line per workload.

--recurrent times kda_recurrent_fwd at the decode workload's shape (256 sequences,
32 heads, d = 128, bf16, per-channel gates) for each token count T, next to T calls
of kda_decode_step on the same inputs, with the algorithmic bytes of
roofline.recurrent_bytes (state read once and written once per call).
"""
from __future__ import annotations

import argparse
import ctypes
import dataclasses
import json
import os
import statistics

import torch

import kimi_delta_attention_22_b200 as kda
from kimi_delta_attention_22_b200 import inputs
from kimi_delta_attention_22_b200.roofline import (backward_bytes, backward_flops, prefill_bytes, prefill_flops,
                                                   recurrent_bytes)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        return json.load(f)


def measure(name: str, schedule: str, iters: int, warmup: int, shape=None) -> dict:
    """shape = (B, T, H): the workload's recipe at other sizes (dense workloads only)."""
    w = inputs.WORKLOADS[name]
    if shape is not None:
        if w.varlen:
            raise ValueError("--shape applies to dense workloads only")
        B, T, H = shape
        w = dataclasses.replace(w, name=f"{name}@B{B}_T{T}_H{H}", B=B, T=T, H=H,
                                qk_heads=(H * w.qk_heads // w.H if w.qk_heads else 0))
    d = inputs.workload_inputs(w, device="cuda")
    cu = d.get("cu_seqlens")
    ws = None
    if schedule == "workspace":
        n = kda.kda_chunk_fwd_workspace_size(d["q"], d["v"], d["g"], cu_seqlens=cu, chunk=w.chunk)
        ws = torch.empty(n, dtype=torch.uint8, device="cuda") if n else None
    out = torch.empty_like(d["v"])
    N = w.num_seqs if w.varlen else w.B
    S_T = torch.empty(N, w.H, w.d_v, w.d_k, dtype=torch.float32, device="cuda")

    def call():
        kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S0=d["S0"], cu_seqlens=cu,
                          chunk=w.chunk, out=out, S_T=S_T, workspace=ws if ws is not None else False)

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    times = []
    for _ in range(iters):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        call()
        b.record(stream)
        b.synchronize()
        times.append(a.elapsed_time(b))
    ms = statistics.median(times)
    nbytes, flops = prefill_bytes(w), prefill_flops(w)
    res = {"workload": w.name, "schedule": schedule, "ms_per_call": ms,
           "tokens_per_s": w.tokens / (ms * 1e-3), "hbm_gbs": nbytes / (ms * 1e-3) / 1e9,
           "tflops": flops / (ms * 1e-3) / 1e12, "algorithmic_bytes": nbytes, "flops": flops,
           "iters": iters}
    pk = peaks()
    if pk:
        res["hbm_frac"] = res["hbm_gbs"] / pk["hbm_gbs"]
        res["tc_frac"] = res["tflops"] / pk["bf16_tflops"]
    del d, ws, out, S_T
    torch.cuda.empty_cache()
    return res


def _time(fn, iters: int, warmup: int) -> float:
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    times = []
    for _ in range(iters):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        times.append(a.elapsed_time(b))
    return statistics.median(times)


def measure_recurrent(T: int, iters: int, warmup: int, N: int = 256, H: int = 32) -> dict:
    d = inputs.draw(N, T, H, 128, 128, dtype=torch.bfloat16, gate="channel", s0_std=0.05, seed=7,
                    device="cuda")
    S = d["S0"].clone()
    out = torch.empty_like(d["v"])
    steps = [{k: d[k][:, t].contiguous() for k in ("q", "k", "v", "g", "beta")} for t in range(T)]
    step_out = torch.empty(N, H, 128, dtype=torch.bfloat16, device="cuda")

    def fused():
        kda.kda_recurrent_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S, out=out)

    def per_token():
        for st in steps:
            kda.kda_decode_step(st["q"], st["k"], st["v"], st["g"], st["beta"], S, out=step_out)

    ms = _time(fused, iters, warmup)
    ms_steps = _time(per_token, iters, warmup)
    nbytes = recurrent_bytes(N, T, H, 128, 128)
    res = {"kernel": "kda_recurrent_fwd", "N": N, "H": H, "T": T, "ms_per_call": ms,
           "tokens_per_s": N * T / (ms * 1e-3), "hbm_gbs": nbytes / (ms * 1e-3) / 1e9,
           "algorithmic_bytes": nbytes, "decode_steps_ms": ms_steps,
           "speedup_vs_decode_steps": ms_steps / ms, "iters": iters}
    pk = peaks()
    if pk:
        res["hbm_frac"] = res["hbm_gbs"] / pk["hbm_gbs"]
    del d, S, out, steps
    torch.cuda.empty_cache()
    return res


def measure_backward(N: int, T: int, H: int, iters: int, warmup: int) -> dict:
    """kda_recurrent_bwd on N sequences x T tokens x H heads (d = 128, bf16 inputs,
    per-channel gate), against the forward pass of the same tokens."""
    d = inputs.draw(N, T, H, 128, 128, dtype=torch.bfloat16, gate="channel", s0_std=0.05, seed=8,
                    device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(9)
    d_out = torch.randn(N, T, H, 128, device="cuda", generator=gen).to(torch.bfloat16)
    d_ST = torch.randn(N, H, 128, 128, device="cuda", generator=gen)
    sh = kda.Shape(N, T, H, 128, 128, N, kda.KDA_BF16, kda.KDA_GATE_CHANNEL, 0, None, H)
    ws = torch.empty(kda.load_library().kda_recurrent_bwd_workspace_size(ctypes.byref(sh)),
                     dtype=torch.uint8, device="cuda")
    S = d["S0"].clone()

    def bwd():
        kda.kda_recurrent_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], d_out, d_ST, workspace=ws)

    def fwd():
        S.copy_(d["S0"])
        kda.kda_recurrent_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S)

    ms = _time(bwd, iters, warmup)
    ms_f = _time(fwd, iters, warmup)
    # fp32 arithmetic per (token, head, state element): the forward twice (decay,
    # prediction, write: 3 FMA-class ops) and the reverse step (9), FMA counted as 2
    flops = N * T * H * 128 * 128 * 2 * (2 * 3 + 9)
    res = {"kernel": "kda_recurrent_bwd", "N": N, "H": H, "T": T, "ms_per_call": ms,
           "tokens_per_s": N * T / (ms * 1e-3), "fp32_tflops": flops / (ms * 1e-3) / 1e12,
           "forward_ms": ms_f, "backward_over_forward": ms / ms_f, "iters": iters}
    del d, d_out, d_ST, ws, S
    torch.cuda.empty_cache()
    return res


def measure_chunk_backward(name: str, iters: int, warmup: int) -> dict:
    """kda_chunk_bwd on a named workload (seeded N(0, 1) d_out and d_ST, the workspace
    allocated once), next to kda_chunk_fwd on the same inputs."""
    w = inputs.WORKLOADS[name]
    d = inputs.workload_inputs(w, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(w.seed + 1000)
    nseq = w.num_seqs if w.varlen else w.B
    d_out = torch.randn(w.B, w.T, w.H, w.d_v, device="cuda", generator=gen).to(w.torch_dtype)
    d_ST = torch.randn(nseq, w.H, w.d_v, w.d_k, device="cuda", generator=gen)
    cu = d["cu_seqlens"]
    gate = {"channel": kda.KDA_GATE_CHANNEL, "scalar": kda.KDA_GATE_SCALAR, "none": kda.KDA_GATE_NONE}[w.gate_mode]
    sh = kda.Shape(w.B, w.T, w.H, w.d_k, w.d_v, nseq, kda.KDA_BF16, gate, w.chunk, None, w.qk_heads)
    ws = torch.empty(kda.load_library().kda_chunk_bwd_workspace_size(ctypes.byref(sh), int(cu is not None)),
                     dtype=torch.uint8, device="cuda")

    def bwd():
        kda.kda_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], d_out, d_ST=d_ST, cu_seqlens=cu,
                          chunk=w.chunk, workspace=ws)

    def fwd():
        kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S0=d["S0"], cu_seqlens=cu, chunk=w.chunk)

    ms = _time(bwd, iters, warmup)
    ms_f = _time(fwd, iters, warmup)
    nbytes, flops = backward_bytes(w), backward_flops(w)
    res = {"kernel": "kda_chunk_bwd", "workload": name, "ms_per_call": ms, "tokens_per_s": w.tokens / (ms * 1e-3),
           "hbm_gbs": nbytes / (ms * 1e-3) / 1e9, "tflops": flops / (ms * 1e-3) / 1e12,
           "algorithmic_bytes": nbytes, "flops": flops, "forward_ms": ms_f,
           "backward_over_forward": ms / ms_f, "iters": iters}
    pk = peaks()
    if pk:
        res["hbm_frac"] = res["hbm_gbs"] / pk["hbm_gbs"]
        res["tc_frac"] = res["tflops"] / pk["bf16_tflops"]
    del d, d_out, d_ST, ws
    torch.cuda.empty_cache()
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workloads", default=",".join(n for n in inputs.WORKLOADS))
    ap.add_argument("--schedule", choices=["workspace", "pool"], default="workspace")
    ap.add_argument("--iters", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--shape", default=None, help="B,T,H: run the named dense workloads' recipe at these sizes")
    ap.add_argument("--recurrent", action="store_true")
    ap.add_argument("--tokens", default="1,4,16,64")
    ap.add_argument("--backward", default=None,
                    help="N,T,H[;N,T,H...]: time kda_recurrent_bwd on these shapes")
    ap.add_argument("--chunk-backward", default=None,
                    help="workload[,workload...]: time kda_chunk_bwd (bf16, d = 128 workloads)")
    args = ap.parse_args()
    if not torch.cuda.is_available():
        raise SystemExit("measure needs a CUDA device")
    kda.load_library()
    if args.chunk_backward:
        for name in args.chunk_backward.split(","):
            print(json.dumps(measure_chunk_backward(name, args.iters, args.warmup)), flush=True)
        return
    if args.backward:
        for spec in args.backward.split(";"):
            N, T, H = (int(x) for x in spec.split(","))
            print(json.dumps(measure_backward(N, T, H, args.iters, args.warmup)), flush=True)
        return
    if args.recurrent:
        for T in (int(x) for x in args.tokens.split(",")):
            print(json.dumps(measure_recurrent(T, args.iters, args.warmup)), flush=True)
        return
    shape = tuple(int(x) for x in args.shape.split(",")) if args.shape else None
    for name in args.workloads.split(","):
        print(json.dumps(measure(name, args.schedule, args.iters, args.warmup, shape)), flush=True)


if __name__ == "__main__":
    main()
