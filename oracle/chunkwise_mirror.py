"""Float64 numpy restatement of the chunkwise KDA form.  TEST INFRASTRUCTURE ONLY.

The GeekNews summary of "You could have come up with Kimi Delta Attention"
(section "Chunkwise KDA: rearranging the recurrence into matrix products")
states that a chunk of C tokens must reproduce the token loop's states and
outputs exactly, and builds the chunk result from:

  * cumulative decay from the chunk start, inclusive of token i
    (subsection "cumulative decay and provisional errors"):
        Gamma_i = sum_{s<=i} g_s,   D_{0:i} = Diag(exp(Gamma_i)),
    a write of token j reaches token i through D_{j+1:i} = exp(Gamma_i - Gamma_j);
  * provisional errors that ignore the chunk's own writes:
        ebar_i = beta_i (v_i - S_c D_{0:i} k_i);
  * coupling coefficients (subsection "restoring the causal dependency"):
        rho_ij = beta_i k_j^T D_{j+1:i} k_i.

The page stops in the middle of the next formula.  The plainest completion,
used here and by the CUDA kernels, is
    e_i = ebar_i - sum_{j<i} rho_ij e_j        ((I + L) E = Ebar, L strictly lower),
which the curriculum page (objective "pseudo-values from a triangular solve")
names a triangular solve.  The chunk's outputs read the post-write state (the
read step o_t = S_t q~_t), so the in-chunk sum of the output is inclusive (j <= i):
    o_i = S_c D_{0:i} q~_i + sum_{j<=i} (k_j^T D_{j+1:i} q~_i) e_j,
and the outgoing state is
    S_{c+1} = S_c D_{0:C-1} + sum_j e_j k_j^T D_{j+1:C-1}.

This mirror is only a debugging aid that localises a GPU mismatch to the
algorithm or to the kernel; tests check it against the token-loop oracle.
It is plain numpy with no blocking inside a chunk.
"""
from __future__ import annotations

import numpy as np


def chunk_forward_one_pair(q, k, v, g, beta, S0, chunk):
    """One (sequence, head): q,k [T,dk], v [T,dv], g [T,dk] (log alpha, already
    broadcast to every channel), beta [T], S0 [dv,dk].  Returns (o [T,dv], S_T)."""
    q, k, v, g, beta = (np.asarray(a, dtype=np.float64) for a in (q, k, v, g, beta))
    T, dk = k.shape
    S = np.array(S0, dtype=np.float64, copy=True)
    qs = q / np.sqrt(dk)
    out = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, chunk):
        sl = slice(c0, min(c0 + chunk, T))
        K, Q, V, G, b = k[sl], qs[sl], v[sl], g[sl], beta[sl]
        C = K.shape[0]
        Gam = np.cumsum(G, axis=0)                       # Gamma_i, inclusive
        # decay between tokens: R[i, j, c] = exp(Gamma_ic - Gamma_jc) for j <= i
        diff = Gam[:, None, :] - Gam[None, :, :]
        lower = np.tril(np.ones((C, C), dtype=bool))
        R = np.where(lower[:, :, None], np.exp(np.where(lower[:, :, None], diff, 0.0)), 0.0)
        rho = b[:, None] * np.einsum("jc,ijc,ic->ij", K, R, K)
        L = np.tril(rho, -1)                             # strictly lower coupling
        ebar = b[:, None] * (V - (K * np.exp(Gam)) @ S.T)
        E = np.linalg.solve(np.eye(C) + L, ebar)         # (I + L) E = Ebar
        Aqk = np.einsum("jc,ijc,ic->ij", K, R, Q)        # inclusive, j <= i
        out[sl] = (Q * np.exp(Gam)) @ S.T + Aqk @ E
        last = Gam[-1]
        S = S * np.exp(last)[None, :] + E.T @ (K * np.exp(last[None, :] - Gam))
    return out, S


def chunk_forward(q, k, v, g, beta, S0=None, chunk=16, gate="channel"):
    """Dense batch: q,k [B,T,H,dk], v [B,T,H,dv], g per gate mode, beta [B,T,H],
    S0 [B,H,dv,dk] or None.  Returns (out, S_T) in float64."""
    q, k, v, beta = (np.asarray(a, dtype=np.float64) for a in (q, k, v, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if gate == "channel":
        gfull = np.asarray(g, dtype=np.float64)
    elif gate == "scalar":
        gfull = np.repeat(np.asarray(g, dtype=np.float64)[..., None], dk, axis=-1)
    else:
        gfull = np.zeros((B, T, H, dk))
    out = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dv, dk))
    for bi in range(B):
        for h in range(H):
            s0 = np.zeros((dv, dk)) if S0 is None else np.asarray(S0, dtype=np.float64)[bi, h]
            o, s = chunk_forward_one_pair(q[bi, :, h], k[bi, :, h], v[bi, :, h],
                                          gfull[bi, :, h], beta[bi, :, h], s0, chunk)
            out[bi, :, h] = o
            ST[bi, h] = s
    return out, ST
