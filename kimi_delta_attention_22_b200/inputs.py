"""Seeded synthetic inputs for the KDA workloads.

This module holds no KDA arithmetic: it only draws random tensors with the
distributions below, so both the CUDA path and the float64 oracle can be fed
the same values.  Recipe (per token and head):

  * q, k, v ~ N(0, 1), drawn in fp32; k is L2-normalised over d_k in fp32
    (the pages assume normalised keys) and only then cast to the input dtype.
  * beta = sigmoid(N(0, 1))  (or exactly 1.0 in the beta=1 regimes).
  * gate g = log(alpha):
      "channel":        g = -softplus(N(0, 1)) per key channel, so alpha in (0, 1);
      "channel_strong": g = -Uniform(0, 5) per key channel;
      "channel_extreme": g = -Uniform(0, 10) per key channel (close to the largest
                        per-token decay the tensor-core paths hold exactly);
      "scalar":         g = -softplus(N(0, 1)) per (token, head), one value for all channels;
      "none":           no gate (alpha = 1).
  * S0 ~ N(0, s0_std^2) in fp32, or absent (zero state).

Draw order is fixed (q, k, v, g, beta, S0) so a seed names one input set.
Draws use a torch.Generator on the requested device; a given seed therefore
gives different values on CPU and GPU, but every consumer of one generated set
sees the same tensors.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    H: int
    d_k: int
    d_v: int
    dtype: str          # "f32" | "bf16" (q, k, v and out)
    gate: str           # "channel" | "channel_strong" | "channel_extreme" | "scalar" | "none"
    beta: str           # "sigmoid" | "one"
    chunk: int
    s0_std: float | None
    seed: int
    varlen: bool = False
    num_seqs: int = 0   # varlen only
    len_lo: int = 0
    len_hi: int = 0
    qk_heads: int = 0   # query/key heads (grouped value heads); 0 = one per value head

    @property
    def Hk(self) -> int:
        return self.qk_heads or self.H

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def gate_mode(self) -> str:
        return "channel" if self.gate.startswith("channel") else self.gate

    @property
    def tokens(self) -> int:
        return self.B * self.T


WORKLOADS: dict[str, Workload] = {}


def _add(w: Workload):
    WORKLOADS[w.name] = w


# fp32 small case: B=1, H=1, T=64, d=16, chunk 16, zero initial state.
_add(Workload("small_f32_t64_d16", 1, 64, 1, 16, 16, "f32", "channel", "sigmoid", 16, None, 1))
# bf16 chunkwise prefill: B=4, H=16, T=2048, d=128, chunk 64, S0 ~ N(0, 0.02^2).
_add(Workload("prefill_b4_h16_t2048", 4, 2048, 16, 128, 128, "bf16", "channel", "sigmoid", 64,
              0.02, 2))
# the same prefill with grouped value heads: 16 value heads over 4 query/key heads
_add(Workload("prefill_b4_h16_qk4_t2048", 4, 2048, 16, 128, 128, "bf16", "channel", "sigmoid", 64,
              0.02, 12, qk_heads=4))
# varlen prefill: 8 packed sequences, 65536 tokens, lengths in [1024, 15360], state reset.
_add(Workload("varlen_h32_t65536", 1, 65536, 32, 128, 128, "bf16", "channel", "sigmoid", 64,
              None, 4, varlen=True, num_seqs=8, len_lo=1024, len_hi=15360))
# gate-regime sweep at B=8, H=64, T=8192, d=128.
for _gi, _gate in enumerate(("none", "scalar", "channel_strong")):
    for _bi, _beta in enumerate(("one", "sigmoid")):
        _add(Workload(f"sweep_b8_h64_t8192_{_gate}_beta{_beta}", 8, 8192, 64, 128, 128, "bf16",
                      _gate, _beta, 64, None, 50 + 2 * _gi + _bi))

# decode: one token per call for batch 256, H=32, d=128, 128 calls; the state
# comes from a 512-token prefill of the same distributions.
DECODE = dict(name="decode_n256_h32_d128", N=256, H=32, d_k=128, d_v=128, steps=128,
              prefill_T=512, seed=3)


def varlen_lengths(num_seqs: int, total: int, lo: int, hi: int, seed: int) -> list[int]:
    """num_seqs-1 lengths uniform in [lo, hi], the last one takes the rest;
    redraw (same seeded stream) until the last one is in range too."""
    rng = np.random.default_rng(seed)
    while True:
        head = rng.integers(lo, hi + 1, size=num_seqs - 1)
        last = total - int(head.sum())
        if lo <= last <= hi:
            return [int(x) for x in head] + [last]


def _gen(device, seed):
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return gen


def draw(B, T, H, d_k, d_v, *, dtype=torch.bfloat16, gate="channel", beta="sigmoid",
         s0_std=None, num_states=None, seed=0, device="cpu", qk_heads=None):
    """Draw one input set.  Returns a dict with q, k ([B,T,Hk,d_k]), v ([B,T,H,d_v])
    in dtype, g (fp32 [B,T,H,d_k] | [B,T,H] | None), beta (fp32 [B,T,H]) and S0
    (fp32 [num_states,H,d_v,d_k] or None; num_states defaults to B).  Hk =
    qk_heads (grouped value heads) or H."""
    gen = _gen(device, seed)
    f32 = dict(dtype=torch.float32, device=device, generator=gen)
    Hk = H if qk_heads is None else qk_heads
    q = torch.randn(B, T, Hk, d_k, **f32)
    k = torch.randn(B, T, Hk, d_k, **f32)
    k = k / k.norm(dim=-1, keepdim=True).clamp_min(1e-12)
    v = torch.randn(B, T, H, d_v, **f32)
    if gate == "channel":
        g = -torch.nn.functional.softplus(torch.randn(B, T, H, d_k, **f32))
    elif gate == "channel_strong":
        g = -5.0 * torch.rand(B, T, H, d_k, **f32)
    elif gate == "channel_extreme":
        g = -10.0 * torch.rand(B, T, H, d_k, **f32)
    elif gate == "scalar":
        g = -torch.nn.functional.softplus(torch.randn(B, T, H, **f32))
    elif gate == "none":
        g = None
    else:
        raise ValueError(gate)
    if beta == "sigmoid":
        b = torch.sigmoid(torch.randn(B, T, H, **f32))
    elif beta == "one":
        b = torch.ones(B, T, H, dtype=torch.float32, device=device)
    else:
        raise ValueError(beta)
    S0 = None
    if s0_std is not None:
        S0 = s0_std * torch.randn(num_states or B, H, d_v, d_k, **f32)
    return dict(q=q.to(dtype).contiguous(), k=k.to(dtype).contiguous(),
                v=v.to(dtype).contiguous(), g=None if g is None else g.contiguous(), beta=b,
                S0=S0)


def workload_inputs(w: Workload | str, device="cpu", T: int | None = None, B: int | None = None,
                    H: int | None = None):
    """Inputs of a named workload (optionally with B, T or H overridden for a
    smaller case of the same recipe).  Varlen workloads add cu_seqlens (int32,
    on `device`) and use a leading batch of 1."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    B_, T_, H_ = B or w.B, T or w.T, H or w.H
    out = draw(B_, T_, H_, w.d_k, w.d_v, dtype=w.torch_dtype, gate=w.gate, beta=w.beta,
               s0_std=w.s0_std, seed=w.seed, device=device,
               num_states=(w.num_seqs if w.varlen else None),
               qk_heads=(H_ * w.qk_heads // w.H if w.qk_heads else None))
    out["cu_seqlens"] = None
    if w.varlen:
        lo = max(1, w.len_lo * T_ // w.T)
        hi = max(lo, w.len_hi * T_ // w.T)
        lens = varlen_lengths(w.num_seqs, T_, lo, hi, w.seed)
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        out["cu_seqlens"] = torch.from_numpy(cu).to(device)
    return out


def decode_inputs(N, H, d_k, d_v, steps, seed, device="cpu", dtype=torch.bfloat16,
                  gate="channel"):
    """Per-step decode inputs: q,k [steps,N,H,d_k], v [steps,N,H,d_v],
    g [steps,N,H,d_k], beta [steps,N,H] (same recipe as prefill)."""
    d = draw(steps, N, H, d_k, d_v, dtype=dtype, gate=gate, seed=seed, device=device)
    return d
