"""Benchmark of the KDA hot path on B200.

One step = one kda_chunk_fwd call over the bf16 prefill workload (B=4, H=16,
T=2048, d_k=d_v=128, chunk 64, per-channel gates, S0 ~ N(0, 0.02^2)): every
chunkwise step (cumulative decay, decay-masked products, triangular solve,
state scan and outputs) runs inside that one call (the WY, sub-block WY and
state-scan kernels over a preallocated workspace; --schedule pool: the same
kernels with no workspace passed, so each call takes its scratch from the
stream-ordered memory pool).  After it, reported as extra objects of the same
line: "e2e" (the same step from pinned host buffers, copies included),
"no_workspace" (the same call without a workspace), "varlen" (8 packed
sequences, 65,536 tokens, 32 heads) and "sweep" (B=8, H=64, T=8192 in six
gate / beta regimes), each with its own roofline; "decode" (256 x 32 heads,
d=128, fp32 state in HBM, 128 one-token calls after a 512-token prefill),
"backward" (kda_chunk_bwd, the chunkwise gradients of the prefill workload,
with its own roofline) and "backward_recurrent" (kda_recurrent_bwd, 256 x 32
heads x 16 tokens).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line on rank 0.  Under torchrun each rank runs its own
replica (weak scaling; the path has no exchange step).  The reference arm
(--impl reference) times the float64 CPU oracle on the host cores.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch

from kimi_delta_attention_22_b200.roofline import backward_bytes, backward_flops, prefill_bytes, prefill_flops

METRIC = "KDA prefill tokens/s (% bf16 TC peak); decode step HBM GB/s (% of peak)"
WORKLOAD = "prefill_b4_h16_t2048"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_HBM_GBS = 7700.0   # nominal HBM3e bandwidth of one B200 (context for fractions of the copy peak)
_CSRC = "kimi_delta_attention_22_b200/csrc/"
PREFILL_SRC = [_CSRC + f for f in ("kda_chunk_wy.cu", "kda_chunk_scan.cu", "kda_chunk_scan.cuh",
                                   "kda_chunk_record.cuh", "kda_tc_common.cuh", "sm100.cuh")]
CHUNK_BWD_SRC = PREFILL_SRC + [_CSRC + f for f in ("kda_chunk_bwd.cuh", "kda_chunk_bwd_scan.cu",
                                                   "kda_chunk_bwd_grad.cu")]


# ------------------------------------------------------------------ helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_sha(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def dram_traffic(kernel_tag, workload, src_paths):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on
    the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(p):
        return None
    sha = source_sha(src_paths)
    with open(p) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel_tag and \
                    parts[1] == workload and parts[2] == sha:
                return float(parts[3])
    return None


class ClockSampler:
    """nvidia-smi clock / throttle sampling in the background."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        # nvidia-smi numbers GPUs physically; address this process's GPU by UUID
        try:
            self.idx = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            self.idx = str(device_index)
        self.proc = None
        self.path = f"/tmp/kda_bench_clocks_{os.getpid()}.csv"

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}",
                                          f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) >= 10:
                    rows.append(p)
        os.unlink(self.path)
        busy = [r for r in rows if r[4].isdigit() and int(r[4]) > 0] or rows
        sm = [float(r[1]) for r in busy if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in busy for i in range(4) if r[6 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "samples_busy": len(busy)}


def init_dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64,
                     device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------- CPU (oracle)

def oracle_prefill(d, nthreads=0):
    import oracle

    t0 = time.perf_counter()
    oracle.forward(d["q"], d["k"], d["v"], d["g"], d["beta"], S0=d["S0"], nthreads=nthreads)
    return time.perf_counter() - t0


def cpu_inputs(w, seed_offset=0):
    from kimi_delta_attention_22_b200 import inputs

    return inputs.draw(w.B, w.T, w.H, w.d_k, w.d_v, dtype=w.torch_dtype, gate=w.gate,
                       beta=w.beta, s0_std=w.s0_std, seed=w.seed + seed_offset, device="cpu")


def run_reference(args, world, rank):
    """--impl reference: the float64 oracle on the host cores, each step the
    whole prefill workload (64 (sequence, head) pairs x 2048 tokens)."""
    from kimi_delta_attention_22_b200 import inputs

    import oracle

    if rank != 0:
        return
    w = inputs.WORKLOADS[WORKLOAD]
    d = cpu_inputs(w)
    cores = oracle.max_threads()
    for _ in range(args.warmup):
        oracle_prefill(d)
    times = [oracle_prefill(d) for _ in range(args.steps)]
    total = sum(times)
    val = args.steps * w.tokens / total
    line = {"metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD, "B": w.B, "T": w.T, "H": w.H, "d_k": w.d_k,
                       "d_v": w.d_v, "chunk": w.chunk, "gate": w.gate, "parallelism": "none"},
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"whole workload per step ({w.B * w.H} (sequence, head) "
                                       f"pairs x {w.T} tokens), float64 token loop"},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU path

def bench_prefill(args, world, rank, peaks, peak_kind):
    import kimi_delta_attention_22_b200 as kda
    from kimi_delta_attention_22_b200 import inputs

    kda.load_library()
    w = inputs.WORKLOADS[WORKLOAD]
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    n_sets = 3  # rotating input sets (3 x ~210 MB > 126 MB L2): no step re-reads from L2
    sets = [inputs.draw(w.B, w.T, w.H, w.d_k, w.d_v, dtype=w.torch_dtype, gate=w.gate,
                        beta=w.beta, s0_std=w.s0_std, seed=w.seed + 100 * rank + i, device=dev)
            for i in range(n_sets)]
    outs = [torch.empty_like(s["v"]) for s in sets]
    STs = [torch.empty(w.B, w.H, w.d_v, w.d_k, dtype=torch.float32, device=dev) for _ in sets]
    # scratch of the two-kernel schedule, allocated once outside the timed region
    # (--schedule pool: no workspace, each call draws it from the stream-ordered pool)
    ws = None if args.schedule == "pool" else torch.empty(
        kda.kda_chunk_fwd_workspace_size(sets[0]["q"], sets[0]["v"], sets[0]["g"], chunk=w.chunk),
        dtype=torch.uint8, device=dev)

    def step(i):
        s = sets[i % n_sets]
        kda.kda_chunk_fwd(s["q"], s["k"], s["v"], s["g"], s["beta"], S0=s["S0"], chunk=w.chunk,
                          out=outs[i % n_sets], S_T=STs[i % n_sets], workspace=ws)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        step(i)
        ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    elapsed_ms = max_over_ranks(t0.elapsed_time(t1), world)
    launch_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    launch_ms = max_over_ranks(launch_ms, world)

    alg_bytes = prefill_bytes(w)
    flops = prefill_flops(w)
    achieved_gbs = alg_bytes / (launch_ms * 1e-3) / 1e9
    achieved_tf = flops / (launch_ms * 1e-3) / 1e12
    traffic = dram_traffic("chunk_fwd", WORKLOAD, PREFILL_SRC)
    res = {
        "w": w, "elapsed_ms": elapsed_ms, "launch_ms": launch_ms,
        "value": world * args.steps * w.tokens / (elapsed_ms * 1e-3),
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved_gbs / peaks["hbm_gbs"],
                     "traffic": traffic, "peak_source": f"{peak_kind} hbm_gbs",
                     "algorithmic_bytes_per_launch": alg_bytes,
                     "kernel": "kda_chunk_fwd call (WY, sub-block WY and state-scan kernels)"},
        "tensor": {"achieved_tflops": achieved_tf, "flops_per_launch": flops,
                   "peak_tflops": peaks["bf16_tflops"],
                   "frac": achieved_tf / peaks["bf16_tflops"],
                   "peak_source": f"{peak_kind} bf16_tflops (burst)"},
    }
    # ---- the same call with no workspace: the scratch comes from the stream-ordered
    #      pool (cudaMallocAsync / cudaFreeAsync on the call's stream) every call
    nw_iters = max(5, min(args.steps, 20))
    for i in range(2):
        s = sets[i % n_sets]
        kda.kda_chunk_fwd(s["q"], s["k"], s["v"], s["g"], s["beta"], S0=s["S0"], chunk=w.chunk,
                          out=outs[i % n_sets], S_T=STs[i % n_sets], workspace=None)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(nw_iters):
        s = sets[i % n_sets]
        kda.kda_chunk_fwd(s["q"], s["k"], s["v"], s["g"], s["beta"], S0=s["S0"], chunk=w.chunk,
                          out=outs[i % n_sets], S_T=STs[i % n_sets], workspace=None)
    b.record(stream)
    torch.cuda.synchronize()
    nw_ms = max_over_ranks(a.elapsed_time(b), world) / nw_iters
    res["no_workspace"] = {"ms_per_call": nw_ms, "iters": nw_iters,
                           "value": world * w.tokens / (nw_ms * 1e-3), "unit": "tokens/s",
                           "vs_workspace": nw_ms / (elapsed_ms / args.steps),
                           "scratch": "cudaMallocAsync / cudaFreeAsync on the call's stream"}
    # ---- end to end through the public API with host buffers: every step copies
    #      its inputs from pinned host memory, runs the call and reads out and S_T
    #      back, all inside the timed region.  Steps are double-buffered on three
    #      streams (H2D, compute, D2H) as a serving loop would be, so the copies of
    #      one step overlap the call and the copies of its neighbours.
    host = {k: (None if v is None else v.cpu().pin_memory()) for k, v in sets[0].items()}
    dbufs = [sets[1], sets[2]]
    hout = torch.empty(outs[0].shape, dtype=outs[0].dtype).pin_memory()
    hST = torch.empty(STs[0].shape, dtype=torch.float32).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = hout.numel() * hout.element_size() + hST.numel() * 4
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    ready = [ev(), ev()]      # inputs of buffer b landed
    done = [ev(), ev()]       # the call on buffer b finished (its inputs and outputs are free
    drained = [ev(), ev()]    # outputs of buffer b read back      ... once drained)
    for b in range(2):
        done[b].record(stream)
        drained[b].record(stream)

    def e2e_step(i):
        b = i & 1
        d = dbufs[b]
        with torch.cuda.stream(s_in):
            s_in.wait_event(done[b])
            for k, v in host.items():
                if v is not None:
                    d[k].copy_(v, non_blocking=True)
            ready[b].record(s_in)
        stream.wait_event(ready[b])
        stream.wait_event(drained[b])
        kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S0=d["S0"], chunk=w.chunk,
                          out=outs[1 + b], S_T=STs[1 + b], workspace=ws)
        done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done[b])
            hout.copy_(outs[1 + b], non_blocking=True)
            hST.copy_(STs[1 + b], non_blocking=True)
            drained[b].record(s_out)

    e2e_steps = max(3, min(args.steps, 50))
    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    s_in.wait_stream(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    stream.wait_stream(s_out)
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(a.elapsed_time(b), world) / e2e_steps
    res["e2e"] = {"value": world * w.tokens / (e2e_ms * 1e-3), "unit": "tokens/s",
                  "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                  "steps": e2e_steps, "overlap": "double-buffered H2D / call / D2H streams"}
    del sets, outs, STs, dbufs, ws
    torch.cuda.empty_cache()
    return res


def bench_workload(name, world, peaks, peak_kind, iters=5, warmup=2):
    """One named workload of the larger configurations: inputs drawn once on the
    device (larger than L2), the workspace allocated once, `warmup` untimed calls,
    then `iters` calls back to back between two CUDA events."""
    import kimi_delta_attention_22_b200 as kda
    from kimi_delta_attention_22_b200 import inputs

    w = inputs.WORKLOADS[name]
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    d = inputs.workload_inputs(w, device=dev)
    cu = d.get("cu_seqlens")
    ws = torch.empty(kda.kda_chunk_fwd_workspace_size(d["q"], d["v"], d["g"], cu_seqlens=cu, chunk=w.chunk),
                     dtype=torch.uint8, device=dev)
    out = torch.empty_like(d["v"])
    N = w.num_seqs if w.varlen else w.B
    S_T = torch.empty(N, w.H, w.d_v, w.d_k, dtype=torch.float32, device=dev)

    def call():
        kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S0=d["S0"], cu_seqlens=cu,
                          chunk=w.chunk, out=out, S_T=S_T, workspace=ws)

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(iters):
        call()
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(a.elapsed_time(b), world) / iters
    nbytes, flops = prefill_bytes(w), prefill_flops(w)
    gbs, tf = nbytes / (ms * 1e-3) / 1e9, flops / (ms * 1e-3) / 1e12
    del d, ws, out, S_T
    torch.cuda.empty_cache()
    return {"workload": name, "ms_per_call": ms, "iters": iters,
            "value": world * w.tokens / (ms * 1e-3), "unit": "tokens/s",
            "config": {"B": w.B, "T": w.T, "H": w.H, "gate": w.gate, "beta": w.beta,
                       "varlen": w.varlen, "num_seqs": N},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "peak_source": f"{peak_kind} hbm_gbs",
                         "algorithmic_bytes_per_launch": nbytes,
                         "traffic": dram_traffic("chunk_fwd", name, PREFILL_SRC)},
            "tensor": {"achieved_tflops": tf, "flops_per_launch": flops, "peak_tflops": peaks["bf16_tflops"],
                       "frac": tf / peaks["bf16_tflops"], "peak_source": f"{peak_kind} bf16_tflops (burst)"},
            "gpu_launches": 3 * iters + (1 if w.varlen else 0) * iters}


def bench_chunk_backward(args, world, peaks, peak_kind):
    """kda_chunk_bwd (the chunkwise gradients) on the prefill workload: 4 x 16 heads
    x 2048 tokens, d = 128, chunk 64, per-channel gate; seeded N(0, 1) d_out and d_ST.
    Three rotating input sets (each ~500 MB with its gradients) keep steps out of L2."""
    import kimi_delta_attention_22_b200 as kda
    from kimi_delta_attention_22_b200 import inputs

    w = inputs.WORKLOADS[WORKLOAD]
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    sets = []
    for i in range(3):
        d = inputs.draw(w.B, w.T, w.H, w.d_k, w.d_v, dtype=w.torch_dtype, gate=w.gate, beta=w.beta,
                        s0_std=w.s0_std, seed=w.seed + 200 + i, device=dev)
        gen = torch.Generator(device=dev).manual_seed(300 + i)
        d["d_out"] = torch.randn(w.B, w.T, w.H, w.d_v, device=dev, generator=gen).to(w.torch_dtype)
        d["d_ST"] = torch.randn(w.B, w.H, w.d_v, w.d_k, device=dev, generator=gen)
        sets.append(d)
    sh = kda.Shape(w.B, w.T, w.H, w.d_k, w.d_v, w.B, kda.KDA_BF16, kda.KDA_GATE_CHANNEL, w.chunk, None, 0)
    ws = torch.empty(kda.load_library().kda_chunk_bwd_workspace_size(ctypes.byref(sh), 0),
                     dtype=torch.uint8, device=dev)

    def step(i):
        s = sets[i % 3]
        return kda.kda_chunk_bwd(s["q"], s["k"], s["v"], s["g"], s["beta"], s["S0"], s["d_out"],
                                 d_ST=s["d_ST"], chunk=w.chunk, workspace=ws)

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    iters = 6
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(iters):
        step(i)
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(a.elapsed_time(b), world) / iters
    del sets, ws
    torch.cuda.empty_cache()
    nbytes, flops = backward_bytes(w), backward_flops(w)
    gbs, tf = nbytes / (ms * 1e-3) / 1e9, flops / (ms * 1e-3) / 1e12
    return {"metric": "KDA chunkwise backward tokens/s", "value": world * w.tokens / (ms * 1e-3),
            "unit": "tokens/s", "ms_per_call": ms, "iters": iters,
            "config": {"workload": WORKLOAD, "B": w.B, "T": w.T, "H": w.H, "d_k": w.d_k, "d_v": w.d_v,
                       "chunk": w.chunk, "gate": w.gate, "dtype": "bf16 inputs, fp32 gradients",
                       "l2": "3 rotating input sets > 126 MB L2"},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "peak_source": f"{peak_kind} hbm_gbs",
                         "algorithmic_bytes_per_launch": nbytes,
                         "traffic": dram_traffic("chunk_bwd", WORKLOAD, CHUNK_BWD_SRC),
                         "kernel": "kda_chunk_bwd call (WY, forward scan with checkpoints beside the "
                                   "reverse state scan, solve and dq/dk kernels)"},
            "tensor": {"achieved_tflops": tf, "flops_per_launch": flops, "peak_tflops": peaks["bf16_tflops"],
                       "frac": tf / peaks["bf16_tflops"], "peak_source": f"{peak_kind} bf16_tflops (burst)"},
            "kernels": "kda_chunk_wy_kernel, kda_chunk_fwdbwd_scan_kernel, kda_chunk_bwd_solve_kernel, "
                       "kda_chunk_bwd_dqk_kernel",
            # per call: the two WY kernels, the paired scans, the solve and dq/dk kernels
            "gpu_launches": 5 * iters}


def bench_backward(args, world):
    """kda_recurrent_bwd (gradients of the token loop) on the short-run shape:
    256 sequences x 32 heads x 16 tokens, d = 128, bf16 inputs, per-channel gate."""
    import kimi_delta_attention_22_b200 as kda
    from kimi_delta_attention_22_b200 import inputs

    N, T, H = 256, 16, 32
    dev = torch.device("cuda", torch.cuda.current_device())
    d = inputs.draw(N, T, H, 128, 128, dtype=torch.bfloat16, gate="channel", s0_std=0.05, seed=8, device=dev)
    gen = torch.Generator(device=dev).manual_seed(9)
    d_out = torch.randn(N, T, H, 128, device=dev, generator=gen).to(torch.bfloat16)
    d_ST = torch.randn(N, H, 128, 128, device=dev, generator=gen)
    sh = kda.Shape(N, T, H, 128, 128, N, kda.KDA_BF16, kda.KDA_GATE_CHANNEL, 0, None, H)
    ws = torch.empty(kda.load_library().kda_recurrent_bwd_workspace_size(ctypes.byref(sh)),
                     dtype=torch.uint8, device=dev)

    def step():
        kda.kda_recurrent_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], d_out, d_ST, workspace=ws)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    barrier(world)
    stream = torch.cuda.current_stream(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    iters = 5
    a.record(stream)
    for _ in range(iters):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(a.elapsed_time(b), world) / iters
    del d, d_out, d_ST, ws
    torch.cuda.empty_cache()
    return {"metric": "KDA token-loop backward tokens/s", "value": world * N * T / (ms * 1e-3),
            "unit": "tokens/s", "ms_per_call": ms, "iters": iters,
            "config": {"workload": "recurrent_bwd_n256_h32_t16", "N": N, "T": T, "H": H, "d_k": 128,
                       "d_v": 128, "gate": "channel", "dtype": "bf16 inputs, fp32 gradients"},
            "kernel": "kda_recurrent_bwd_kernel (CUDA cores)"}


def bench_decode(args, world, rank, peaks, peak_kind):
    import kimi_delta_attention_22_b200 as kda
    from kimi_delta_attention_22_b200 import inputs

    D = inputs.DECODE
    N, H, dk, dv, steps = D["N"], D["H"], D["d_k"], D["d_v"], D["steps"]
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    pre = inputs.draw(N, D["prefill_T"], H, dk, dv, seed=D["seed"] + 7 * rank, device=dev)
    _, S = kda.kda_chunk_fwd(pre["q"], pre["k"], pre["v"], pre["g"], pre["beta"])
    del pre
    dec = inputs.decode_inputs(N, H, dk, dv, steps, D["seed"] + 1000 + rank, device=dev)
    out = torch.empty(N, H, dv, dtype=torch.bfloat16, device=dev)
    for t in range(args.warmup):
        kda.kda_decode_step(dec["q"][t], dec["k"][t], dec["v"][t], dec["g"][t], dec["beta"][t], S,
                            out=out)
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for t in range(steps):
        kda.kda_decode_step(dec["q"][t], dec["k"][t], dec["v"][t], dec["g"][t], dec["beta"][t], S,
                            out=out)
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    us = max_over_ranks(a.elapsed_time(b), world) * 1e3 / steps
    state_bytes = N * H * dv * dk * 4
    per_step = 2 * state_bytes + N * H * (2 * (2 * dk + dv) + 4 * dk + 4)
    gbs = per_step / (us * 1e-6) / 1e9
    # some state lines are still in the 126 MB L2 from the previous step, so the
    # algorithmic bytes over the copy peak can exceed 1; frac_spec divides by the nominal
    # HBM3e bandwidth instead, and the ncu DRAM bytes of the same step sit in "traffic"
    del dec, S
    torch.cuda.empty_cache()
    return {"metric": "decode step HBM GB/s", "value": world * gbs, "unit": "GB/s",
            "us_per_step": us, "steps": steps,
            "config": {"workload": D["name"], "N": N, "H": H, "d_k": dk, "d_v": dv,
                       "state_MB": state_bytes / 1e6, "state_from": f"{D['prefill_T']}-token prefill"},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "peak_source": f"{peak_kind} hbm_gbs",
                         "frac_spec": gbs / SPEC_HBM_GBS,
                         "frac_note": "above 1 when state lines stay in L2 between steps",
                         "algorithmic_bytes_per_launch": per_step,
                         "traffic": dram_traffic("decode", D["name"],
                                                 ["kimi_delta_attention_22_b200/csrc/kda_decode.cu"]),
                         "kernel": "kda_decode_kernel"},
            "gpu_launches": steps}


def run_ours(args, world, rank, local):
    peaks, peak_kind = load_peaks()
    clocks = ClockSampler(local)
    clocks.start()
    pre = bench_prefill(args, world, rank, peaks, peak_kind)
    big = {}
    if not args.quick:
        big["varlen"] = bench_workload("varlen_h32_t65536", world, peaks, peak_kind)
        big["sweep"] = [bench_workload(f"sweep_b8_h64_t8192_{g}_beta{b}", world, peaks, peak_kind)
                        for g in ("none", "scalar", "channel_strong") for b in ("one", "sigmoid")]
    dec = bench_decode(args, world, rank, peaks, peak_kind)
    cbwd = bench_chunk_backward(args, world, peaks, peak_kind)
    bwd = bench_backward(args, world)
    clk = clocks.stop()
    w = pre["w"]
    cpu = None
    if rank == 0 and world == 1:
        import oracle

        d = cpu_inputs(w)
        secs = oracle_prefill(d)
        cpu = {"value": w.tokens / secs, "unit": "tokens/s", "cores": oracle.max_threads(),
               "kind": "oracle",
               "sample": f"whole prefill workload once ({w.B * w.H} (sequence, head) pairs x "
                         f"{w.T} tokens, {secs:.1f} s wall), float64 token loop, OpenMP over pairs"}
    if rank == 0:
        line = {"metric": METRIC, "value": pre["value"], "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": pre["elapsed_ms"] / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded N(0,1) q/k/v, L2-normalised k, sigmoid beta, "
                        "-softplus gates)",
                "config": {"workload": WORKLOAD, "B": w.B, "T": w.T, "H": w.H, "d_k": w.d_k,
                           "d_v": w.d_v, "chunk": w.chunk, "gate": w.gate,
                           "global_batch": w.B * world, "seq_len": w.T,
                           "parallelism": f"replicas x{world}",
                           "l2": "3 rotating input sets (~630 MB) > 126 MB L2"},
                "roofline": pre["roofline"], "tensor": pre["tensor"], "cpu_baseline": cpu,
                "e2e": pre["e2e"], "no_workspace": pre["no_workspace"], **big,
                "decode": dec, "backward": cbwd, "backward_recurrent": bwd, "clocks": clk,
                # per step: the WY kernel, the (empty when every chunk takes one reference)
                # sub-block WY kernel and the state scan
                "gpu_launches": 3 * args.steps,
                "schedule": ("two-kernel (parallel WY records + sequential state scan), "
                             + ("scratch from the stream-ordered pool" if args.schedule == "pool"
                                else "preallocated workspace")),
                "kernel_ms_per_launch": pre["launch_ms"]}
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--schedule", choices=["workspace", "pool"], default="workspace",
                    help="prefill scratch: a preallocated workspace (default) or none (stream-ordered pool)")
    ap.add_argument("--quick", action="store_true",
                    help="skip the varlen and sweep workloads")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = init_dist()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            if not torch.cuda.is_available():
                raise SystemExit("bench.py --impl ours needs a CUDA device")
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
