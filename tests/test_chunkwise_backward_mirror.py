"""The chunkwise backward, derived by hand in the float64 mirror
(oracle/chunkwise_mirror.py, chunk_backward), equals autograd of the token loop
(oracle/backward.py) for every gate mode, several chunk sizes with a ragged
last chunk, grouped value heads, and with S0 / d_ST absent.  It fixes the
formulas a chunkwise tensor-core backward would follow: the reverse state
scan, the adjoint of the triangular solve and the decay-weighted Gram
gradients feeding dGamma, then dg as a reverse cumulative sum."""
import numpy as np
import pytest

from oracle import backward as ob
from oracle import chunkwise_mirror as cm


def _inputs(seed, B=2, T=11, H=2, Hk=1, dk=6, dv=5, gate="channel", s0=True, dst=True):
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
    S0 = 0.3 * r.standard_normal((B, H, dv, dk)) if s0 else None
    d_out = r.standard_normal((B, T, H, dv))
    d_ST = r.standard_normal((B, H, dv, dk)) if dst else None
    return dict(q=q, k=k, v=v, g=g, beta=beta, S0=S0, d_out=d_out, d_ST=d_ST)


def _compare(d, chunk, gate):
    ref = ob.backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], d["d_out"], d["d_ST"],
                      gate=gate)
    got = cm.chunk_backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], d["d_out"],
                            d["d_ST"], chunk=chunk, gate=gate)
    for n in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        if ref[n] is None:
            assert got[n] is None, n
            continue
        r = ref[n].numpy()
        assert got[n].shape == r.shape, n
        assert np.max(np.abs(got[n] - r)) <= 1e-12 * max(1.0, np.max(np.abs(r))), n


@pytest.mark.parametrize("gate", ["channel", "scalar", "none"])
@pytest.mark.parametrize("chunk", [1, 4, 16])
def test_chunk_backward_equals_autograd(gate, chunk):
    _compare(_inputs(10 + chunk, gate=gate), chunk, gate)


def test_chunk_backward_grouped_heads_no_state():
    _compare(_inputs(7, H=4, Hk=2, s0=False, dst=False), 4, "channel")


def test_chunk_backward_strong_decay():
    d = _inputs(8, T=20)
    d["g"] = -5.0 * np.random.default_rng(9).random(d["g"].shape)
    _compare(d, 8, "channel")


@pytest.mark.parametrize("chunk", [1, 8, 16])
def test_reverse_state_scan_from_records_alone(chunk):
    """The sequential part of the chunkwise backward needs only the forward's
    record operands (W, Qg, Kd, lower(Qp), gamma): its dS0 equals autograd's."""
    d = _inputs(20 + chunk, B=1, T=37, H=1)
    ref = ob.backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], d["d_out"], d["d_ST"])
    recs = cm.chunk_records_one_pair(d["k"][0, :, 0], d["q"][0, :, 0], d["g"][0, :, 0],
                                     d["beta"][0, :, 0], chunk)
    dS0 = cm.reverse_state_scan(recs, d["d_out"][0, :, 0], d["d_ST"][0, 0])
    r = ref["dS0"].numpy()[0, 0]
    assert np.max(np.abs(dS0 - r)) <= 1e-12 * max(1.0, np.max(np.abs(r)))
