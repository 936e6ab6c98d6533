"""Checks that pin the float64 oracle to facts fixed by the pages and by
mathematics, independent of the oracle's own code.

Each pin is a function ``pin_*(lib)`` that raises AssertionError on failure;
``lib`` selects the compiled oracle (None = the real one), so the same pins can
be run against deliberately broken copies of the oracle (test_oracle_mutants).

Sources ("You could have come up with Kimi Delta Attention": the article's
KDA update; its GeekNews summary, topic 31925):
  * readback after a write: (1 - beta) S~ k + beta v, exactly v when beta = 1 on
    a unit key (GeekNews, "DeltaNet: writing the prediction error");
  * locality: a query orthogonal to the written key is unchanged (same section);
  * I - beta k k^T has eigenvalue 1 - beta on k and 1 on k-perp
    (GeekNews, "structured state transition");
  * one gradient step of size beta on 1/2 ||S k - v||^2 equals the update
    (GeekNews, "deriving it from a reconstruction loss");
  * scalar gate = Gated DeltaNet, no gate = DeltaNet, forget before predict
    (GeekNews, "Gated DeltaNet" and "Kimi Delta Attention");
  * diagonal-plus-low-rank form S_t = S_{t-1} A_t + beta v k^T with
    A_t = D_t - (D_t k_t)(beta_t k_t)^T (GeekNews, "diagonal-plus-low-rank
    transition"), used for an exact-rational brute force on tiny inputs;
  * a hand-worked two-token example (tests/golden/worked_example_d4_t2.json).
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TOL = 1e-12


def _rng(seed):
    return np.random.default_rng(seed)


def _inputs(rng, B, T, H, dk, dv, gate="channel", beta=None, strong=False):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    if gate == "channel":
        g = -rng.uniform(0, 5, (B, T, H, dk)) if strong else -np.log1p(np.exp(rng.standard_normal((B, T, H, dk))))
    elif gate == "scalar":
        g = -np.log1p(np.exp(rng.standard_normal((B, T, H))))
    else:
        g = None
    b = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H)))) if beta is None else np.full((B, T, H), float(beta))
    return q, k, v, g, b


def _close(a, b, tol=TOL, what=""):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} > {tol:.1e} * {scale:.3g}"


# --------------------------------------------------------------------------- pins

def pin_golden_worked_example(lib=None):
    """Hand-worked rational example (worked_example_d4_t2.json)."""
    with open(os.path.join(GOLDEN, "worked_example_d4_t2.json")) as f:
        ex = json.load(f)
    I = ex["inputs"]
    sh = lambda a, d: np.asarray(a, dtype=np.float64).reshape(1, 2, 1, d)
    g = np.log(np.asarray(I["alpha"], dtype=np.float64)).reshape(1, 2, 1, 4)
    beta = np.asarray(I["beta"], dtype=np.float64).reshape(1, 2, 1)
    S0 = np.asarray(I["S0"], dtype=np.float64).reshape(1, 1, 2, 4)
    out, ST = oracle.forward(sh(I["q"], 4), sh(I["k"], 4), sh(I["v"], 2), g, beta, S0=S0,
                             lib=lib)
    _close(out.reshape(2, 2), ex["expected"]["out"], what="golden out")
    _close(ST.reshape(2, 4), ex["expected"]["S_T"], what="golden S_T")


def pin_exact_readback_beta1(lib=None):
    """beta=1 on a unit key: right after the write, reading with k_t returns v_t
    exactly, whatever the decay and the earlier state (the error is measured on
    the decayed state S~)."""
    rng = _rng(11)
    B, T, H, dk, dv = 2, 6, 2, 8, 5
    q, k, v, g, _ = _inputs(rng, B, T, H, dk, dv)
    S0 = rng.standard_normal((B, H, dv, dk))
    out, _ = oracle.forward(k * math.sqrt(dk), k, v, g, np.ones((B, T, H)), S0=S0, lib=lib)
    _close(out, v, tol=1e-12, what="S_t k_t == v_t")


def pin_readback_partial_beta(lib=None):
    """Readback after the write is (1 - beta) S~_t k_t + beta v_t with
    S~_t = S_{t-1} Diag(alpha_t): forget comes before predict."""
    rng = _rng(12)
    B, T, H, dk, dv = 1, 5, 2, 6, 7
    q, k, v, g, b = _inputs(rng, B, T, H, dk, dv)
    S0 = rng.standard_normal((B, H, dv, dk))
    out, _ = oracle.forward(k * math.sqrt(dk), k, v, g, b, S0=S0, lib=lib)
    for t in range(T):
        if t == 0:
            Sprev = S0
        else:
            _, Sprev = oracle.forward(q[:, :t], k[:, :t], v[:, :t], g[:, :t], b[:, :t], S0=S0,
                                      lib=lib)
        for h in range(H):
            Sd = Sprev[0, h] * np.exp(g[0, t, h])[None, :]
            expect = (1 - b[0, t, h]) * (Sd @ k[0, t, h]) + b[0, t, h] * v[0, t, h]
            _close(out[0, t, h], expect, tol=1e-11, what=f"readback t={t} h={h}")


def pin_locality_orthogonal_query(lib=None):
    """No gate (DeltaNet): a query orthogonal to the written key reads the
    same value before and after the write."""
    rng = _rng(13)
    B, T, H, dk, dv = 1, 4, 1, 8, 6
    q, k, v, _, b = _inputs(rng, B, T, H, dk, dv, gate="none")
    S0 = rng.standard_normal((B, H, dv, dk))
    # make q_t orthogonal to k_t
    q = q - np.sum(q * k, axis=-1, keepdims=True) * k
    out, _ = oracle.forward(q, k, v, None, b, S0=S0, gate="none", lib=lib)
    for t in range(T):
        Sprev = S0 if t == 0 else oracle.forward(q[:, :t], k[:, :t], v[:, :t], None, b[:, :t],
                                                 S0=S0, gate="none", lib=lib)[1]
        expect = Sprev[0, 0] @ (q[0, t, 0] / math.sqrt(dk))
        _close(out[0, t, 0], expect, tol=1e-11, what=f"locality t={t}")


def pin_eigenstructure(lib=None):
    """With v = 0 and no gate, one step is S_t = S_{t-1}(I - beta k k^T): the
    transition scales k by 1 - beta and leaves every u orthogonal to k alone."""
    rng = _rng(14)
    dk, dv = 9, 4
    k = rng.standard_normal(dk)
    k /= np.linalg.norm(k)
    S0 = rng.standard_normal((1, 1, dv, dk))
    for beta in (0.0, 0.3, 1.0, 1.7):
        _, S1 = oracle.forward(np.zeros((1, 1, 1, dk)), k.reshape(1, 1, 1, dk),
                               np.zeros((1, 1, 1, dv)), None, np.full((1, 1, 1), beta), S0=S0,
                               gate="none", lib=lib)
        _close(S1[0, 0] @ k, (1 - beta) * (S0[0, 0] @ k), tol=1e-12, what="eigen on k")
        for _ in range(3):
            u = rng.standard_normal(dk)
            u -= (u @ k) * k
            _close(S1[0, 0] @ u, S0[0, 0] @ u, tol=1e-12, what="eigen on k-perp")


def pin_online_gradient_step(lib=None):
    """No gate: S_t = S_{t-1} - beta * grad_S 1/2 ||S k - v||^2 at S_{t-1}, with the
    gradient taken by central differences (exact for a quadratic up to rounding)."""
    rng = _rng(15)
    dk, dv = 5, 3
    S0 = rng.standard_normal((dv, dk))
    k = rng.standard_normal(dk)
    k /= np.linalg.norm(k)
    v = rng.standard_normal(dv)
    beta = 0.37
    loss = lambda S: 0.5 * float(np.sum((S @ k - v) ** 2))
    grad = np.zeros_like(S0)
    h = 1e-3
    for r in range(dv):
        for c in range(dk):
            E = np.zeros_like(S0)
            E[r, c] = h
            grad[r, c] = (loss(S0 + E) - loss(S0 - E)) / (2 * h)
    _, S1 = oracle.forward(np.zeros((1, 1, 1, dk)), k.reshape(1, 1, 1, dk), v.reshape(1, 1, 1, dv),
                           None, np.full((1, 1, 1), beta), S0=S0.reshape(1, 1, dv, dk),
                           gate="none", lib=lib)
    _close(S1[0, 0], S0 - beta * grad, tol=1e-9, what="online GD step")


def pin_pure_decay(lib=None):
    """beta = 0: nothing is written, so S_t = S0 Diag(exp(sum_{s<=t} g_s)) and
    o_t = S_t q~_t (closed form; d_k != d_v catches a transposed Diag)."""
    rng = _rng(16)
    B, T, H, dk, dv = 2, 7, 3, 6, 4
    q, k, v, g, _ = _inputs(rng, B, T, H, dk, dv)
    S0 = rng.standard_normal((B, H, dv, dk))
    out, ST = oracle.forward(q, k, v, g, np.zeros((B, T, H)), S0=S0, lib=lib)
    Gam = np.cumsum(g, axis=1)
    for bi in range(B):
        for h in range(H):
            _close(ST[bi, h], S0[bi, h] * np.exp(Gam[bi, -1, h])[None, :], what="decay S_T")
            for t in range(T):
                St = S0[bi, h] * np.exp(Gam[bi, t, h])[None, :]
                _close(out[bi, t, h], St @ q[bi, t, h] / math.sqrt(dk), what="decay out")


def pin_scalar_gate_pure_decay(lib=None):
    """Scalar gate, beta = 0: S_T = S0 * prod_t alpha_t (Gated DeltaNet forget)."""
    rng = _rng(17)
    B, T, H, dk, dv = 1, 5, 2, 4, 3
    q, k, v, g, _ = _inputs(rng, B, T, H, dk, dv, gate="scalar")
    S0 = rng.standard_normal((B, H, dv, dk))
    _, ST = oracle.forward(q, k, v, g, np.zeros((B, T, H)), S0=S0, gate="scalar", lib=lib)
    for h in range(H):
        _close(ST[0, h], S0[0, h] * math.exp(float(np.sum(g[0, :, h]))), what="scalar decay")


def pin_zero_inputs(lib=None):
    """v = 0 and S0 = 0 leave the state and every output at zero."""
    rng = _rng(18)
    B, T, H, dk, dv = 1, 6, 2, 8, 8
    q, k, v, g, b = _inputs(rng, B, T, H, dk, dv)
    out, ST = oracle.forward(q, k, np.zeros_like(v), g, b, lib=lib)
    assert np.all(out == 0) and np.all(ST == 0), "zero inputs give nonzero result"


def _dplr_bruteforce(q, k, v, alpha, beta, S0):
    """Exact rationals: S_t = S_{t-1} A_t + beta_t v_t k_t^T with
    A_t = D_t - (D_t k_t)(beta_t k_t)^T; o_t = S_t q_t / sqrt(d_k) (d_k a square)."""
    T, dk = k.shape
    dv = v.shape[1]
    root = math.isqrt(dk)
    assert root * root == dk
    Fr = lambda x: Fraction(float(x))
    S = [[Fr(S0[r, c]) for c in range(dk)] for r in range(dv)]
    outs = []
    for t in range(T):
        a = [Fr(x) for x in alpha[t]]
        kk = [Fr(x) for x in k[t]]
        b = Fr(beta[t])
        A = [[(a[i] if i == j else Fraction(0)) - a[i] * kk[i] * b * kk[j] for j in range(dk)]
             for i in range(dk)]
        S = [[sum(S[r][i] * A[i][j] for i in range(dk)) + b * Fr(v[t, r]) * kk[j]
              for j in range(dk)] for r in range(dv)]
        qs = [Fr(x) / root for x in q[t]]
        outs.append([sum(S[r][c] * qs[c] for c in range(dk)) for r in range(dv)])
    return np.array([[float(x) for x in o] for o in outs]), np.array([[float(x) for x in row] for row in S])


def pin_dplr_bruteforce_exact(lib=None):
    """Exact-rational brute force of the diagonal-plus-low-rank product form on
    T <= 8 tokens, d_k in {4, 16}; the float64 oracle must agree to 1e-12."""
    for seed, (T, dk, dv) in enumerate([(8, 4, 3), (5, 16, 2), (3, 4, 4)]):
        rng = _rng(100 + seed)
        q, k, v, g, b = _inputs(rng, 1, T, 1, dk, dv)
        S0 = rng.standard_normal((1, 1, dv, dk))
        alpha = np.exp(g[0, :, 0])  # the same float64 values the oracle forms
        out, ST = oracle.forward(q, k, v, g, b, S0=S0, lib=lib)
        eo, es = _dplr_bruteforce(q[0, :, 0], k[0, :, 0], v[0, :, 0], alpha, b[0, :, 0], S0[0, 0])
        _close(out[0, :, 0], eo, what=f"brute force out T={T} dk={dk}")
        _close(ST[0, 0], es, what=f"brute force S_T T={T} dk={dk}")


def pin_gate_modes_consistent(lib=None):
    """A scalar gate equals a per-channel gate with that value on every channel,
    and no gate equals a per-channel gate of zeros."""
    rng = _rng(19)
    B, T, H, dk, dv = 2, 6, 2, 8, 5
    q, k, v, gs, b = _inputs(rng, B, T, H, dk, dv, gate="scalar")
    S0 = rng.standard_normal((B, H, dv, dk))
    o1, s1 = oracle.forward(q, k, v, gs, b, S0=S0, gate="scalar", lib=lib)
    o2, s2 = oracle.forward(q, k, v, np.repeat(gs[..., None], dk, -1), b, S0=S0, lib=lib)
    _close(o1, o2, what="scalar vs channel out")
    _close(s1, s2, what="scalar vs channel S_T")
    o3, s3 = oracle.forward(q, k, v, None, b, S0=S0, gate="none", lib=lib)
    o4, s4 = oracle.forward(q, k, v, np.zeros((B, T, H, dk)), b, S0=S0, lib=lib)
    _close(o3, o4, what="none vs zero gate out")
    _close(s3, s4, what="none vs zero gate S_T")


def pin_resume_and_varlen(lib=None):
    """Splitting a sequence and resuming from S_T equals one pass; packed
    sequences with cu_seqlens equal separate calls."""
    rng = _rng(20)
    T, H, dk, dv = 9, 2, 6, 5
    q, k, v, g, b = _inputs(rng, 1, T, H, dk, dv)
    S0 = rng.standard_normal((1, H, dv, dk))
    o, s = oracle.forward(q, k, v, g, b, S0=S0, lib=lib)
    o1, s1 = oracle.forward(q[:, :4], k[:, :4], v[:, :4], g[:, :4], b[:, :4], S0=S0, lib=lib)
    o2, s2 = oracle.forward(q[:, 4:], k[:, 4:], v[:, 4:], g[:, 4:], b[:, 4:], S0=s1, lib=lib)
    _close(np.concatenate([o1, o2], axis=1), o, what="resume out")
    _close(s2, s, what="resume S_T")
    lens = [3, 0, 6]
    cu = np.concatenate([[0], np.cumsum(lens)])
    S0v = rng.standard_normal((3, H, dv, dk))
    ov, sv = oracle.forward(q, k, v, g, b, S0=S0v, cu_seqlens=cu, lib=lib)
    for n in range(3):
        sl = slice(cu[n], cu[n + 1])
        if lens[n] == 0:
            _close(sv[n], S0v[n], what="empty sequence keeps S0")
            continue
        on, sn = oracle.forward(q[:, sl], k[:, sl], v[:, sl], g[:, sl], b[:, sl],
                                S0=S0v[n:n + 1], lib=lib)
        _close(ov[:, sl], on, what=f"varlen out seq {n}")
        _close(sv[n], sn[0], what=f"varlen S_T seq {n}")


def pin_linearity_and_causality(lib=None):
    """For fixed q, k, g, beta the map (S0, v) -> (out, S_T) is linear, and
    out_t does not depend on tokens after t."""
    rng = _rng(21)
    B, T, H, dk, dv = 1, 7, 2, 6, 5
    q, k, v, g, b = _inputs(rng, B, T, H, dk, dv)
    v2 = rng.standard_normal(v.shape)
    S0a, S0b = rng.standard_normal((2, B, H, dv, dk))
    oa, sa = oracle.forward(q, k, v, g, b, S0=S0a, lib=lib)
    ob, sb = oracle.forward(q, k, v2, g, b, S0=S0b, lib=lib)
    oc, sc = oracle.forward(q, k, 2 * v - 3 * v2, g, b, S0=2 * S0a - 3 * S0b, lib=lib)
    _close(oc, 2 * oa - 3 * ob, tol=1e-11, what="linearity out")
    _close(sc, 2 * sa - 3 * sb, tol=1e-11, what="linearity S_T")
    q2, k2, v3, g2, b2 = _inputs(_rng(22), B, T, H, dk, dv)
    for a, a2 in ((q, q2), (k, k2), (v, v3), (g, g2), (b, b2)):
        a[:, 4:] = a2[:, 4:]
    od, _ = oracle.forward(q, k, v, g, b, S0=S0a, lib=lib)
    _close(od[:, :4], oa[:, :4], tol=0.0, what="causality")


def pin_chunkwise_identity(lib=None):
    """The chunkwise form (cumulative decay, coupling, triangular solve) gives
    the token loop's states and outputs for any chunk size, ragged tail included."""
    from oracle import chunkwise_mirror

    for strong in (False, True):
        rng = _rng(23 + strong)
        B, T, H, dk, dv = 1, 70, 2, 8, 6
        q, k, v, g, b = _inputs(rng, B, T, H, dk, dv, strong=strong)
        S0 = rng.standard_normal((B, H, dv, dk))
        o, s = oracle.forward(q, k, v, g, b, S0=S0, lib=lib)
        for C in (1, 2, 4, 16, 64):
            oc, sc = chunkwise_mirror.chunk_forward(q, k, v, g, b, S0=S0, chunk=C)
            _close(oc, o, tol=1e-10, what=f"chunk C={C} out strong={strong}")
            _close(sc, s, tol=1e-10, what=f"chunk C={C} S_T strong={strong}")


def pin_grouped_value_heads(lib=None):
    """Grouped value heads: G consecutive value heads share one query/key head
    (the value-head grid axis of the fused recurrent kernel in the GeekNews
    summary).  Equal, bit for bit, to the one-to-one recurrence with each q/k
    head repeated for its G value heads; a mapping that pairs value head h with
    q/k head h mod Hk (or ignores the grouping) differs."""
    rng = _rng(41)
    B, T, Hk, G, dk, dv = 2, 6, 2, 3, 4, 5
    H = Hk * G
    q = rng.standard_normal((B, T, Hk, dk))
    k = rng.standard_normal((B, T, Hk, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    g = -np.log1p(np.exp(rng.standard_normal((B, T, H, dk))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    S0 = 0.1 * rng.standard_normal((B, H, dv, dk))
    o1, s1 = oracle.forward(q, k, v, g, beta, S0=S0, gate="channel", lib=lib)
    o2, s2 = oracle.forward(np.repeat(q, G, axis=2), np.repeat(k, G, axis=2), v, g, beta, S0=S0,
                            gate="channel", lib=lib)
    assert np.array_equal(o1, o2) and np.array_equal(s1, s2), "grouped value heads != repeated q/k"
    # value heads of different groups must see different q/k heads
    o3, _ = oracle.forward(np.repeat(q[:, :, ::-1], G, axis=2), np.repeat(k[:, :, ::-1], G, axis=2), v,
                           g, beta, S0=S0, gate="channel", lib=lib)
    assert not np.allclose(o1, o3)


ALL_PINS = [v for n, v in sorted(globals().items()) if n.startswith("pin_")]
