"""Algorithmic work of one kda_chunk_fwd call on a named workload, the
numerators of the roofline fractions that bench.py and measure.py report.

Bytes: every input read once and every output written once (per head-token
q, k, v, out at the input element size, g at 4 bytes per channel / per token /
none, beta 4 bytes; S0 and S_T at 4 bytes per state element per sequence).
FLOPs (multiply-add = 2): the chunkwise form at chunk C, counting only the
causal halves of the in-chunk products."""
from __future__ import annotations


def prefill_bytes(w) -> int:
    """q and k count once per query/key head (grouped value heads share them)."""
    ht = w.B * w.T * w.H
    Hk = getattr(w, "Hk", w.H)
    el = 2 if w.dtype == "bf16" else 4
    g = {"channel": 4 * w.d_k, "scalar": 4, "none": 0}[w.gate_mode]
    per_ht = el * w.d_v + g + 4 + el * w.d_v
    qk = w.B * w.T * Hk * el * 2 * w.d_k
    seqs = w.num_seqs if w.varlen else w.B
    states = seqs * w.H * w.d_v * w.d_k * 4 * ((1 if w.s0_std is not None else 0) + 1)
    return ht * per_ht + qk + states


def prefill_flops(w) -> float:
    """Per head-token at chunk C: A_kk and A_qk 2*C*d_k (causal halves); W and U
    C*(d_k + d_v); E = U - W S^T 2*d_k*d_v; O = Q S^T + A_qk E 2*d_k*d_v + C*d_v;
    state update 2*d_k*d_v; triangular solve C^2/3."""
    C, dk, dv = w.chunk, w.d_k, w.d_v
    per_ht = (2 * C * dk) + (C * dk + C * dv) + 2 * dk * dv + (2 * dk * dv + C * dv) + \
        2 * dk * dv + C * C / 3.0
    return w.B * w.T * w.H * per_ht


def recurrent_bytes(N: int, T: int, H: int, d_k: int, d_v: int, el: int = 2, gate: str = "channel") -> int:
    """Algorithmic HBM bytes of one kda_recurrent_fwd call: the fp32 state read
    once and written once, plus every token's q, k, v, out (el bytes), g and beta."""
    g = {"channel": 4 * d_k, "scalar": 4, "none": 0}[gate]
    per_ht = el * (2 * d_k + 2 * d_v) + g + 4
    return 2 * N * H * d_v * d_k * 4 + N * T * H * per_ht


def backward_bytes(w) -> int:
    """Algorithmic HBM bytes of one kda_chunk_bwd call: every input read once
    (q, k, v, d_out at the input element size, g, beta, S0 and d_ST) and every
    gradient written once in fp32 (dq, dk per query/key head; dv, dg, dbeta per
    value head; dS0 per sequence and head)."""
    ht = w.B * w.T * w.H
    Hk = getattr(w, "Hk", w.H)
    el = 2 if w.dtype == "bf16" else 4
    g = {"channel": 4 * w.d_k, "scalar": 4, "none": 0}[w.gate_mode]
    per_ht = 2 * el * w.d_v + 2 * g + 4 + 4 + 4 * w.d_v          # v, d_out, g + dg, beta + dbeta, dv
    qk = w.B * w.T * Hk * 2 * w.d_k * (el + 4)                    # q, k and dq, dk
    seqs = w.num_seqs if w.varlen else w.B
    states = seqs * w.H * w.d_v * w.d_k * 4 * ((1 if w.s0_std is not None else 0) + 2)
    return ht * per_ht + qk + states


def backward_flops(w) -> float:
    """The forward recomputed (prefill_flops), then per head-token at chunk C:
    the reverse state scan 6*d_k*d_v + C*d_v (dE = Kd dS'^T + lower(Qp)^T dO and
    dS <- dS Diag + dO^T Qg - dE^T W); the solve half 2*d_k*d_v + 3*C*d_v + C*d_k
    (the residual product, E, dEbar and dL over their causal halves, the key Gram);
    the dq/dk half 6*d_k*d_v + C*d_v + 4*C*d_k (dKd, dQg, dKg, dAqk and the two
    decay-weighted Grams' gradients)."""
    C, dk, dv = w.chunk, w.d_k, w.d_v
    per_ht = 14 * dk * dv + 5 * C * dv + 5 * C * dk
    return prefill_flops(w) + w.B * w.T * w.H * per_ht
