"""Pins of the float64 gradient reference (oracle/backward.py), the first step
of the backward pass: its forward equals the C token loop, its gradients equal
central finite differences of the loss, and for one token from a zero state they
equal the closed form (o = beta (k . q~) v)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as ob


def _inputs(seed, B=2, T=5, H=4, Hk=2, dk=6, dv=5, gate="channel"):
    r = np.random.default_rng(seed)
    q = r.standard_normal((B, T, Hk, dk))
    k = r.standard_normal((B, T, Hk, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((B, T, H, dv))
    g = None
    if gate == "channel":
        g = -np.log1p(np.exp(r.standard_normal((B, T, H, dk))))
    elif gate == "scalar":
        g = -np.log1p(np.exp(r.standard_normal((B, T, H))))
    beta = 1.0 / (1.0 + np.exp(-r.standard_normal((B, T, H))))
    S0 = 0.3 * r.standard_normal((B, H, dv, dk))
    return dict(q=q, k=k, v=v, g=g, beta=beta, S0=S0)


@pytest.mark.parametrize("gate", ["channel", "scalar", "none"])
def test_forward_equals_c_oracle(gate):
    d = _inputs(1, gate=gate)
    ro, rs = oracle.forward(d["q"], d["k"], d["v"], d["g"], d["beta"], S0=d["S0"], gate=gate)
    t = {n: (None if x is None else torch.from_numpy(x)) for n, x in d.items()}
    o, s = ob.forward(t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], gate=gate)
    assert np.max(np.abs(o.numpy() - ro)) < 1e-12 and np.max(np.abs(s.numpy() - rs)) < 1e-12


@pytest.mark.parametrize("gate", ["channel", "scalar", "none"])
def test_gradients_equal_finite_differences(gate):
    d = _inputs(2, gate=gate)
    r = np.random.default_rng(3)
    d_out = r.standard_normal(d["v"].shape)
    d_ST = r.standard_normal(d["S0"].shape)
    grads = ob.backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], d_out, d_ST, gate=gate)

    def loss(dd):
        o, s = oracle.forward(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], S0=dd["S0"], gate=gate)
        return float((o * d_out).sum() + (s * d_ST).sum())

    eps = 1e-6
    for name in ("q", "k", "v", "g", "beta", "S0"):
        if d[name] is None:
            assert grads["d" + name] is None
            continue
        gr = grads["d" + name].numpy()
        flat = d[name].reshape(-1)
        for idx in r.choice(flat.size, size=min(6, flat.size), replace=False):
            dp = {n: (None if x is None else x.copy()) for n, x in d.items()}
            dm = {n: (None if x is None else x.copy()) for n, x in d.items()}
            dp[name].reshape(-1)[idx] += eps
            dm[name].reshape(-1)[idx] -= eps
            fd = (loss(dp) - loss(dm)) / (2 * eps)
            an = gr.reshape(-1)[idx]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, an)


def test_one_token_closed_form():
    """T = 1 from a zero state: S = beta v k^T, so o = beta (k . q~) v with
    q~ = q / sqrt(dk); for the loss sum(o * w): dv = beta (k . q~) w,
    dbeta = (k . q~)(v . w), dq = beta (v . w) k / sqrt(dk), dk = beta (v . w) q~."""
    r = np.random.default_rng(4)
    dk, dv = 8, 6
    q, k, v, w = (r.standard_normal((1, 1, 1, n)) for n in (dk, dk, dv, dv))
    beta = np.array([[[0.7]]])
    grads = ob.backward(q, k, v, None, beta, None, w, None, gate="none")
    qs = q[0, 0, 0] / np.sqrt(dk)
    kq, vw = float(k[0, 0, 0] @ qs), float(v[0, 0, 0] @ w[0, 0, 0])
    b = 0.7
    np.testing.assert_allclose(grads["dv"].numpy()[0, 0, 0], b * kq * w[0, 0, 0], atol=1e-13)
    np.testing.assert_allclose(grads["dbeta"].numpy()[0, 0, 0], kq * vw, atol=1e-13)
    np.testing.assert_allclose(grads["dq"].numpy()[0, 0, 0], b * vw * k[0, 0, 0] / np.sqrt(dk), atol=1e-13)
    np.testing.assert_allclose(grads["dk"].numpy()[0, 0, 0], b * vw * qs, atol=1e-13)
    assert grads["dS0"] is None and grads["dg"] is None
