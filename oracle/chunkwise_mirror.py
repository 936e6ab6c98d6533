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

``chunk_backward`` differentiates the same chunk form by hand (the pages give
no backward derivation): a reverse scan over chunks carries dL/dS from each
chunk's outgoing state to its incoming one, and within a chunk every step of
the forward is undone in reverse order -- the state update, the outputs, the
triangular solve (dEbar = (I + L)^-T dE, dL = -dEbar E^T on the strict lower
triangle), the provisional errors, the decay-weighted Gram entries (whose
exp(Gamma_i - Gamma_j) factor feeds dGamma_i and -dGamma_j) and finally the
cumulative sum (dg = reverse cumulative sum of dGamma).  Tests check it
against autograd of the token loop (oracle/backward.py).
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


def _decay_gram_backward(dX, P, K, R):
    """Gradients of X_ij = sum_c P_ic K_jc R_ijc (R_ijc = exp(Gamma_ic - Gamma_jc)
    on the masked entries, 0 elsewhere): returns dP, dK, dGamma."""
    W = dX[:, :, None] * R                       # dX_ij R_ijc
    dP = np.einsum("ijc,jc->ic", W, K)
    dK = np.einsum("ijc,ic->jc", W, P)
    T = W * P[:, None, :] * K[None, :, :]        # dX_ij P_ic K_jc R_ijc
    dGam = T.sum(axis=1) - T.sum(axis=0)
    return dP, dK, dGam


def chunk_backward_one_pair(q, k, v, g, beta, S0, d_out, d_ST, chunk):
    """Gradients of sum(out * d_out) + sum(S_T * d_ST) for one (sequence, head):
    returns dq, dk [T,dk], dv [T,dv], dg [T,dk] (per channel), dbeta [T], dS0."""
    q, k, v, g, beta, d_out = (np.asarray(a, dtype=np.float64) for a in (q, k, v, g, beta, d_out))
    T, dk = k.shape
    dv_ = v.shape[1]
    sq = 1.0 / np.sqrt(dk)
    qs = q * sq
    starts = list(range(0, T, chunk))
    # forward: the incoming state of every chunk
    S_in = []
    S = np.array(S0, dtype=np.float64, copy=True)
    for c0 in starts:
        S_in.append(S.copy())
        _, S = chunk_forward_one_pair(q[c0:c0 + chunk], k[c0:c0 + chunk], v[c0:c0 + chunk],
                                      g[c0:c0 + chunk], beta[c0:c0 + chunk], S, chunk)
    dq, dk_, dv, dg, db = (np.zeros_like(q), np.zeros_like(k), np.zeros_like(v), np.zeros_like(g),
                           np.zeros_like(beta))
    dS = np.zeros((dv_, dk)) if d_ST is None else np.array(d_ST, dtype=np.float64)
    for ci in range(len(starts) - 1, -1, -1):
        sl = slice(starts[ci], min(starts[ci] + chunk, T))
        S = S_in[ci]
        K, Q, V, G, b, dO = k[sl], qs[sl], v[sl], g[sl], beta[sl], d_out[sl]
        C = K.shape[0]
        # ---- forward of the chunk again, keeping the intermediates
        Gam = np.cumsum(G, axis=0)
        lower = np.tril(np.ones((C, C), dtype=bool))
        strict = np.tril(np.ones((C, C), dtype=bool), -1)
        diff = Gam[:, None, :] - Gam[None, :, :]
        R = np.where(lower[:, :, None], np.exp(np.where(lower[:, :, None], diff, 0.0)), 0.0)
        A = np.einsum("jc,ijc,ic->ij", K, R, K)
        L = np.where(strict, b[:, None] * A, 0.0)
        M = np.eye(C) + L
        Kg = K * np.exp(Gam)
        resid = V - Kg @ S.T                     # V - Kg S^T
        ebar = b[:, None] * resid
        E = np.linalg.solve(M, ebar)
        Aqk = np.einsum("jc,ijc,ic->ij", K, R, Q)
        Qg = Q * np.exp(Gam)
        gam = Gam[-1]
        Kd = K * np.exp(gam[None, :] - Gam)
        dSp = dS                                 # dL/d(outgoing state)
        # ---- S' = S Diag(e^gam) + E^T Kd
        dS_in = dSp * np.exp(gam)[None, :]
        dgam = np.einsum("vc,vc->c", S, dSp) * np.exp(gam)
        dE = Kd @ dSp.T
        dKd = E @ dSp
        dK = dKd * np.exp(gam[None, :] - Gam)
        dGam = -dKd * Kd
        dgam += (dKd * Kd).sum(axis=0)
        # ---- O = Qg S^T + Aqk E
        dQg = dO @ S
        dS_in += dO.T @ Qg
        dAqk = np.where(lower, dO @ E.T, 0.0)
        dE += Aqk.T @ dO
        dQ = dQg * np.exp(Gam)
        dGam += dQg * Qg
        dP, dKq, dG2 = _decay_gram_backward(dAqk, Q, K, R)
        dQ += dP
        dK += dKq
        dGam += dG2
        # ---- E = (I + L)^-1 Ebar
        debar = np.linalg.solve(M.T, dE)
        dL = np.where(strict, -debar @ E.T, 0.0)
        # ---- Ebar = b (V - Kg S^T)
        db_c = (debar * resid).sum(axis=1)
        dV = b[:, None] * debar
        dPr = -b[:, None] * debar                # d(Kg S^T)
        dKg = dPr @ S
        dS_in += dPr.T @ Kg
        dK += dKg * np.exp(Gam)
        dGam += dKg * Kg
        # ---- L = strict_lower(b_i A_ij)
        db_c += (dL * A).sum(axis=1)
        dA = b[:, None] * dL
        dP, dKa, dG3 = _decay_gram_backward(dA, K, K, R)
        dK += dP + dKa
        dGam += dG3
        # ---- Gamma = cumsum(G); gam = Gamma_last
        dGam[-1] += dgam
        dG = np.cumsum(dGam[::-1], axis=0)[::-1]
        dq[sl], dk_[sl], dv[sl], dg[sl], db[sl] = dQ * sq, dK, dV, dG, db_c
        dS = dS_in
    return dq, dk_, dv, dg, db, dS


def chunk_backward(q, k, v, g, beta, S0, d_out, d_ST=None, chunk=16, gate="channel"):
    """Dense batch, layouts of chunk_forward (q, k [B,T,Hk,dk] with H a multiple
    of Hk; value head h reads q/k head h // (H // Hk)).  Returns a dict like
    oracle.backward.backward: dq, dk, dv, dg (None without a gate; [B,T,H] for a
    scalar gate), dbeta, dS0, in float64."""
    q, k, v, beta, d_out = (np.asarray(a, dtype=np.float64) for a in (q, k, v, beta, d_out))
    B, T, Hk, dk = q.shape
    H, dv = v.shape[2], v.shape[3]
    grp = H // Hk
    if gate == "channel":
        gfull = np.asarray(g, dtype=np.float64)
    elif gate == "scalar":
        gfull = np.repeat(np.asarray(g, dtype=np.float64)[..., None], dk, axis=-1)
    else:
        gfull = np.zeros((B, T, H, dk))
    res = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v),
               dg=np.zeros((B, T, H, dk)), dbeta=np.zeros_like(beta), dS0=np.zeros((B, H, dv, dk)))
    for bi in range(B):
        for h in range(H):
            hk = h // grp
            s0 = np.zeros((dv, dk)) if S0 is None else np.asarray(S0, dtype=np.float64)[bi, h]
            dST = None if d_ST is None else np.asarray(d_ST, dtype=np.float64)[bi, h]
            gq, gk, gv, gg, gb, gs = chunk_backward_one_pair(
                q[bi, :, hk], k[bi, :, hk], v[bi, :, h], gfull[bi, :, h], beta[bi, :, h], s0,
                d_out[bi, :, h], dST, chunk)
            res["dq"][bi, :, hk] += gq
            res["dk"][bi, :, hk] += gk
            res["dv"][bi, :, h] = gv
            res["dg"][bi, :, h] = gg
            res["dbeta"][bi, :, h] = gb
            res["dS0"][bi, h] = gs
    if gate == "scalar":
        res["dg"] = res["dg"].sum(axis=-1)
    elif gate == "none":
        res["dg"] = None
    if S0 is None:
        res["dS0"] = None
    return res


def chunk_records_one_pair(k, q, g, beta, chunk):
    """Per chunk of one (sequence, head): the state-independent operands the
    forward's WY records hold -- W = T diag(beta) (K e^Gamma), Qg = Q~ e^Gamma,
    Kd = K e^{gamma - Gamma}, lower(Qp) (the inclusive A_qk) and gamma = Gamma_last."""
    k, q, g, beta = (np.asarray(a, dtype=np.float64) for a in (k, q, g, beta))
    T, dk = k.shape
    qs = q / np.sqrt(dk)
    recs = []
    for c0 in range(0, T, chunk):
        sl = slice(c0, min(c0 + chunk, T))
        K, Q, G, b = k[sl], qs[sl], g[sl], beta[sl]
        C = K.shape[0]
        Gam = np.cumsum(G, axis=0)
        lower = np.tril(np.ones((C, C), dtype=bool))
        strict = np.tril(np.ones((C, C), dtype=bool), -1)
        R = np.where(lower[:, :, None],
                     np.exp(np.where(lower[:, :, None], Gam[:, None, :] - Gam[None, :, :], 0.0)), 0.0)
        A = np.einsum("jc,ijc,ic->ij", K, R, K)
        Tinv = np.linalg.inv(np.eye(C) + np.where(strict, b[:, None] * A, 0.0))
        recs.append(dict(rows=sl, W=Tinv @ (b[:, None] * K * np.exp(Gam)), Qg=Q * np.exp(Gam),
                         Kd=K * np.exp(Gam[-1][None, :] - Gam),
                         AQ=np.einsum("jc,ijc,ic->ij", K, R, Q), gamma=Gam[-1]))
    return recs


def reverse_state_scan(recs, d_out, d_ST):
    """dL/dS0 of one (sequence, head) from the records alone, chunk by chunk in
    reverse: dE = Kd dS^T + lower(Qp)^T dO, then
    dS <- dS Diag(e^gamma) + dO^T Qg - dE^T W (using (beta . dEbar)^T K e^Gamma = dE^T W)."""
    d_out = np.asarray(d_out, dtype=np.float64)
    dS = np.array(d_ST, dtype=np.float64, copy=True)
    for r in reversed(recs):
        dO = d_out[r["rows"]]
        dE = r["Kd"] @ dS.T + r["AQ"].T @ dO
        dS = dS * np.exp(r["gamma"])[None, :] + dO.T @ r["Qg"] - dE.T @ r["W"]
    return dS
