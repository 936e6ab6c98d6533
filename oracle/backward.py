"""Float64 gradients of the KDA recurrence -- TEST INFRASTRUCTURE ONLY.

Only ``tests/`` may import this module; the library never does.  The pages name
training as the use of the chunkwise schedule but give no backward derivation,
so the reference for gradients is the definition itself: the token loop of the
five-step update of "You could have come up with Kimi Delta Attention" (the
equations at the top of the article; GeekNews summary, section "Kimi Delta
Attention: per-channel decay"), written with PyTorch float64 CPU tensors, and
differentiated by ``torch.autograd`` (a library primitive).  ``forward`` is the
same loop as ``oracle.forward`` (the C token loop), vectorised over sequences
and heads; tests check the two agree.

Layouts as ``oracle.forward`` (dense batches): q, k [B,T,Hk,dk]; v [B,T,H,dv];
g [B,T,H,dk] (channel) | [B,T,H] (scalar) | None; beta [B,T,H];
S0 [B,H,dv,dk] or None; H a multiple of Hk (value head h reads q/k head
h // (H // Hk)).
"""
from __future__ import annotations

import torch

__all__ = ["forward", "backward"]


def _t(x):
    if x is None:
        return None
    x = torch.as_tensor(x)
    return x.detach().to(device="cpu", dtype=torch.float64).clone()


def forward(q, k, v, g, beta, S0=None, gate="channel"):
    """(out [B,T,H,dv], S_T [B,H,dv,dk]) in float64 for float64 tensor inputs
    (those with requires_grad build the autograd graph)."""
    B, T, Hk, dk = q.shape
    H, dv = v.shape[2], v.shape[3]
    G = H // Hk
    qh = q.repeat_interleave(G, dim=2) if G > 1 else q
    kh = k.repeat_interleave(G, dim=2) if G > 1 else k
    scale = 1.0 / dk ** 0.5
    S = torch.zeros(B, H, dv, dk, dtype=torch.float64) if S0 is None else S0
    outs = []
    for t in range(T):
        kt, qt, vt, bt = kh[:, t], qh[:, t], v[:, t], beta[:, t]
        if gate == "channel":
            alpha = torch.exp(g[:, t])                       # [B,H,dk]
        elif gate == "scalar":
            alpha = torch.exp(g[:, t])[..., None].expand(B, H, dk)
        else:
            alpha = torch.ones(B, H, dk, dtype=torch.float64)
        S = S * alpha[:, :, None, :]                          # forget
        vhat = torch.einsum("bhrc,bhc->bhr", S, kt)           # predict
        e = bt[..., None] * (vt - vhat)                       # correct
        S = S + e[..., :, None] * kt[..., None, :]            # write
        outs.append(torch.einsum("bhrc,bhc->bhr", S, qt * scale))   # read
    return torch.stack(outs, dim=1), S


def backward(q, k, v, g, beta, S0, d_out, d_ST=None, gate="channel"):
    """Gradients of sum(out * d_out) + sum(S_T * d_ST) with respect to every
    input, in float64: dict with dq, dk, dv, dg (None without a gate), dbeta,
    dS0 (None when S0 is None)."""
    ins = {n: _t(x) for n, x in dict(q=q, k=k, v=v, g=g, beta=beta, S0=S0).items()}
    leaves = {n: x.requires_grad_(True) for n, x in ins.items() if x is not None}
    out, ST = forward(ins["q"], ins["k"], ins["v"], ins["g"], ins["beta"], ins["S0"], gate=gate)
    loss = (out * _t(d_out)).sum()
    if d_ST is not None:
        loss = loss + (ST * _t(d_ST)).sum()
    names = list(leaves)
    grads = torch.autograd.grad(loss, [leaves[n] for n in names])
    res = {f"d{n}": None for n in ("q", "k", "v", "g", "beta", "S0")}
    for n, gr in zip(names, grads):
        res[f"d{n}"] = gr
    return res
