"""The decay-factor splits of the tensor-core kernels, emulated on the CPU.

The kernels never form e^{Gamma_i - Gamma_j} directly: they multiply an i-side factor
2^{G_i - G_r} and a j-side factor 2^{G_r - G_j} around a reference row r (G = Gamma in
log2 units), as operands of a product (the chunkwise form's decay-masked Gram, the
GeekNews summary of "You could have come up with Kimi Delta Attention", section
"Chunkwise KDA").  These tests replay that arithmetic in fp32 with the device's
flush-to-zero exp2 and bf16 operand rounding, against float64, and pin the range
arguments the kernels rely on:

* two references (rows 15 and 47, one per 32-row half), taken while every 16-row
  sub-block's decay is <= 100: every operand finite, the Gram close to float64;
* sub-block references, a later sub-block's j-side formed as one power
  2^{G_rI - G_j}: exact for strong decay, where the product of the two powers
  2^{G_rb - G_j} 2^{G_rI - G_rb} loses terms (the second factor underflows);
* the backward's pair factor applied in two steps split at the end of sub-block J.
"""
import numpy as np
import pytest

LOG2E = 1.4426950408889634
FTZ = np.float32(2.0 ** -126)


def ex2(x):
    """exp2 in fp32 with denormal results flushed to zero."""
    y = np.exp2(np.asarray(x, dtype=np.float32)).astype(np.float32)
    return np.where(np.abs(y) < FTZ, np.float32(0), y)


def mul(a, b):
    y = (np.asarray(a, dtype=np.float32) * np.asarray(b, dtype=np.float32)).astype(np.float32)
    return np.where(np.abs(y) < FTZ, np.float32(0), y)


def bf16(x):
    """Round fp32 to bf16 (nearest even), returned as fp32."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32)


def split2(x):
    hi = bf16(x)
    return hi, bf16(np.asarray(x, dtype=np.float32) - hi)


def chunk(seed, scale, C=64, d=32):
    r = np.random.default_rng(seed)
    k = r.standard_normal((C, d))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    g = -scale * r.random((C, d)) if np.isscalar(scale) else scale
    G = np.cumsum(g, axis=0) * LOG2E   # float64, log2 units
    return k.astype(np.float32), G


def gram_true(k, G):
    """P_ij = sum_c k_ic k_jc 2^{G_ic - G_jc} for j < i, float64."""
    C = k.shape[0]
    P = np.zeros((C, C))
    for i in range(C):
        for j in range(i):
            P[i, j] = np.sum(k[i].astype(np.float64) * k[j] * np.exp2(G[i] - G[j]))
    return P


def test_two_reference_gram_is_finite_and_close():
    """Chunks that pass the two-reference test (strong decay, -U(0,5) per token): every
    operand is finite and the Gram, from single-term bf16 rows and two-term j-sides,
    is within 1e-2 of its largest entry."""
    checked = 0
    for seed in range(40):
        k, G = chunk(seed, 5.0)
        Gf = G.astype(np.float32)
        blocks = np.concatenate([[np.zeros(k.shape[1])], G[15::16]])   # G before and at rows 15, 31, 47, 63
        if np.max(blocks[:-1] - blocks[1:]) > 100 or np.max(-G[-1]) <= 112:
            continue   # not a two-reference chunk
        checked += 1
        P = np.zeros((64, 64), dtype=np.float64)
        for h, r in ((0, 15), (1, 47)):
            rows = np.arange(64) if h == 0 else np.arange(32, 64)
            cols = np.arange(32 * h, 32 * h + 32)
            x = ex2(Gf[rows] - Gf[r])      # i-side over r
            y = ex2(Gf[r] - Gf[cols])      # j-side over r
            A = bf16(mul(k[rows], x))
            yh, yl = split2(mul(k[cols], y))
            assert np.all(np.isfinite(A)) and np.all(np.isfinite(yh)) and np.all(np.isfinite(yl))
            with np.errstate(over="ignore", invalid="ignore"):   # entries above the diagonal
                part = A @ yh.T + A @ yl.T
            P[np.ix_(rows, cols)] = part
        ref = gram_true(k, G)
        mask = np.tril(np.ones((64, 64), dtype=bool), -1)
        assert np.all(np.isfinite(P[mask]))
        assert np.max(np.abs(P - ref)[mask]) <= 1e-2 * np.max(np.abs(ref))
    assert checked >= 5


def test_later_subblock_j_side_as_one_power():
    """Sub-block references 16 I + 7, decay 7 nats per token (beyond 16 tokens of which
    the pair factor 2^{G_rI - G_rb} underflows): the one-power j-side keeps the cross-
    sub-block Gram exact; the product of two powers drops it."""
    d = 32
    k, G = chunk(3, np.full((64, d), -7.0), d=d)
    Gf = G.astype(np.float32)
    ref = gram_true(k, G)
    one, two = np.zeros((64, 64)), np.zeros((64, 64))
    for I in range(1, 4):
        rI = 16 * I + 7
        rows = np.arange(16 * I, 16 * I + 16)
        x = ex2(Gf[rows] - Gf[rI])
        for b in range(I):
            rb = 16 * b + 7
            cols = np.arange(16 * b, 16 * b + 16)
            ki = mul(k[rows], x)
            one[np.ix_(rows, cols)] = ki @ mul(k[cols], ex2(Gf[rI] - Gf[cols])).T
            two[np.ix_(rows, cols)] = ki @ mul(mul(k[cols], ex2(Gf[rb] - Gf[cols])), ex2(Gf[rI] - Gf[rb])).T
    cross = np.zeros((64, 64), dtype=bool)
    for I in range(1, 4):
        cross[16 * I:16 * I + 16, :16 * I] = True
    scale = np.max(np.abs(ref[cross]))
    assert scale > 1e-6                                   # the adjacent rows' terms matter
    assert np.max(np.abs(one - ref)[cross]) <= 1e-4 * scale
    assert np.max(np.abs(two - ref)[cross]) >= 0.5 * scale   # the earlier form loses them


def test_backward_pair_factor_in_two_steps():
    """The backward's j-side b_j = 2^{G_rJ - G_j} times the pair factor: applied as
    f1 = 2^{G_m(J) - G_rJ} (m(J) = 16 J + 15) and then f2 = 2^{G_rI - G_m(J)}, the
    cross-sub-block Gram is exact; one factor d = 2^{G_rI - G_rJ} underflows."""
    d = 32
    k, G = chunk(5, np.full((64, d), -7.0), d=d)
    Gf = G.astype(np.float32)
    ref = gram_true(k, G)
    a = np.zeros((64, d), dtype=np.float32)
    b = np.zeros((64, d), dtype=np.float32)
    for I in range(4):
        rows = np.arange(16 * I, 16 * I + 16)
        a[rows] = mul(k[rows], ex2(Gf[rows] - Gf[16 * I + 7]))
        b[rows] = mul(k[rows], ex2(Gf[16 * I + 7] - Gf[rows]))
    steps, single = np.zeros((64, 64)), np.zeros((64, 64))
    cross = np.zeros((64, 64), dtype=bool)
    for I in range(1, 4):
        for J in range(I):
            rows, cols = np.arange(16 * I, 16 * I + 16), np.arange(16 * J, 16 * J + 16)
            f1 = ex2(Gf[16 * J + 15] - Gf[16 * J + 7])
            f2 = ex2(Gf[16 * I + 7] - Gf[16 * J + 15])
            dd = ex2(Gf[16 * I + 7] - Gf[16 * J + 7])
            steps[np.ix_(rows, cols)] = a[rows] @ mul(mul(b[cols], f1), f2).T
            single[np.ix_(rows, cols)] = a[rows] @ mul(b[cols], dd).T
            cross[np.ix_(rows, cols)] = True
    scale = np.max(np.abs(ref[cross]))
    assert np.all(np.isfinite(steps))
    assert np.max(np.abs(steps - ref)[cross]) <= 1e-4 * scale   # fp32 rounding of four factors
    assert np.max(np.abs(single - ref)[cross]) >= 0.5 * scale


@pytest.mark.parametrize("scale", [1.0, 2.4])
def test_one_reference_operands_finite_below_threshold(scale):
    """One reference (the chunk start) while max_c |G_last| <= 112: the j-side
    2^{-G_j} <= 2^112 and the i-side 2^{G_i} >= 2^-112 stay normal, so the bf16
    operands are finite and nonzero for every channel with a nonzero key."""
    for seed in range(20):
        k, G = chunk(100 + seed, scale)
        if np.max(-G[-1]) > 112:
            continue
        Gf = G.astype(np.float32)
        x, y = ex2(Gf), ex2(-Gf)
        assert np.all(np.isfinite(y)) and np.all(x > 0)
