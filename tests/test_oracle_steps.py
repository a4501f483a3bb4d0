"""Pins of the oracle's per-head steps (RMSNorm, NeoX and GPT-J RoPE) against
closed forms, invariants and complex multiplication."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads

D = 128
rng = np.random.default_rng(20240)


# ------------------------------------------------------------------ RMSNorm

@pytest.mark.parametrize("scale", [1e-2, 1.0, 37.0, 1e3])
def test_rmsnorm_unit_weights_mean_square(scale):
    """With w = 1: mean(y^2) = ms / (ms + eps) where ms = mean(x^2)."""
    eps = 1e-6
    for _ in range(20):
        x = (rng.standard_normal(D) * scale).astype(np.float32)
        y = oracle.rmsnorm(x, None, eps).astype(np.float64)
        ms = np.mean(x.astype(np.float64) ** 2)
        assert np.mean(y ** 2) == pytest.approx(ms / (ms + eps), rel=2e-6)


@pytest.mark.parametrize("a", [1e-5, 3e-3, 0.5, 1.0, 7.25, 900.0])
@pytest.mark.parametrize("k", [0, 63, 64, 127])
def test_rmsnorm_one_hot_closed_form(a, k):
    """x = a e_k gives y_k = a / sqrt(a^2 / 128 + eps), zeros elsewhere: the
    divisor is the full head (128) and eps sits inside the square root."""
    eps = 1e-6
    x = np.zeros(D, np.float32)
    x[k] = a
    y = oracle.rmsnorm(x, None, eps)
    want = np.float64(np.float32(a)) / np.sqrt(np.float64(np.float32(a)) ** 2 / 128 + eps)
    assert y[k] == pytest.approx(want, rel=3e-7)
    assert np.all(np.delete(y, k) == 0)


def test_rmsnorm_zero_head_is_zero():
    y = oracle.rmsnorm(np.zeros(D, np.float32), np.ones(D, np.float32), 1e-6)
    assert np.all(y == 0)


@pytest.mark.parametrize("c", [1e-2, 0.125, 3.0, 1e3])
def test_rmsnorm_scale_relation(c):
    """norm(c x) = norm(x) * c * sqrt((ms + eps) / (c^2 ms + eps)); for eps << ms
    this is scale invariance."""
    eps = 1e-6
    x = rng.standard_normal(D).astype(np.float32)
    xc = (x * np.float32(c)).astype(np.float32)
    y1 = oracle.rmsnorm(x, None, eps).astype(np.float64)
    y2 = oracle.rmsnorm(xc, None, eps).astype(np.float64)
    ms = np.mean(x.astype(np.float64) ** 2)
    msc = np.mean(xc.astype(np.float64) ** 2)
    ratio = np.sqrt((ms + eps) / (msc + eps)) * (msc / ms) ** 0.5
    assert np.allclose(y2, y1 * ratio, rtol=2e-6, atol=1e-30)


def _bf16_valued(a):
    """float32 values truncated to BF16 (8 significant bits), as the packed
    rows deliver them."""
    a = np.asarray(a, np.float32)
    return (a.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)


def _round_to_f32(q: Fraction) -> np.float32:
    """Round an exact rational to the nearest binary32 (ties to even), from
    the definition: the quantum of q's binade, an integer count of quanta
    rounded half-to-even, and the result rebuilt (normal range only)."""
    if q == 0:
        return np.float32(0.0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    quantum = Fraction(2) ** (e - 23)
    n, rem = divmod(a, quantum)
    if rem * 2 > quantum or (rem * 2 == quantum and n % 2 == 1):
        n += 1
    return np.float32(sign * float(n * quantum))


@pytest.mark.parametrize("scale", [1e-3, 1.0, 40.0])
def test_rmsnorm_sum_is_order_free(scale):
    """The mean square is a function of the multiset of squares: permuting a
    head's elements permutes its output, bit for bit.  A sequential fp32 sum
    depends on the order and fails this on some of these heads."""
    for _ in range(60):
        x = _bf16_valued(rng.standard_normal(D) * scale)
        y = oracle.rmsnorm(x, None, 1e-6)
        for _ in range(4):
            p = rng.permutation(D)
            assert np.array_equal(oracle.rmsnorm(x[p], None, 1e-6), y[p])


def test_rmsnorm_mean_square_is_the_rounded_exact_mean():
    """y = x * (1 / sqrt(ms + eps)) with ms the binary32 rounding of the exact
    rational mean of the squares (computed here with exact fractions), then
    IEEE fp32 addition, square root and reciprocal."""
    eps = np.float32(1e-6)
    for scale in (1e-2, 0.7, 3.0, 250.0):
        for _ in range(25):
            x = _bf16_valued(rng.standard_normal(D) * scale)
            s = sum(Fraction(float(v)) ** 2 for v in x)
            ms = _round_to_f32(s / D)
            inv = np.float32(1.0) / np.sqrt(np.float32(ms + eps))
            want = (x * inv).astype(np.float32)
            assert np.array_equal(oracle.rmsnorm(x, None, float(eps)), want)


def test_rmsnorm_large_element_beside_small_ones():
    """x = (4096, 1, ..., 1): the squares sum to 2^24 + 127 exactly, which a
    running fp32 sum rounds away to 2^24 (every +1 is lost), shifting y_0 by
    about 3.8e-6 relative.  The closed form of the exact mean square is
    y_0 = 4096 / sqrt((2^24 + 127) / 128 + eps)."""
    x = np.ones(D, np.float32)
    x[0] = 4096.0
    y = oracle.rmsnorm(x, None, 1e-6).astype(np.float64)
    ms = (2.0 ** 24 + 127) / 128
    assert y[0] == pytest.approx(4096 / np.sqrt(ms + 1e-6), rel=2.5e-7)
    assert y[1] == pytest.approx(1 / np.sqrt(ms + 1e-6), rel=2.5e-7)


def test_rmsnorm_weight_applies_after_normalisation():
    """norm(x, w) equals norm(x) times w element by element, and differs from
    normalising x * w (the weight must not enter the mean square)."""
    x = rng.standard_normal(D).astype(np.float32)
    w = (1 + 0.5 * rng.standard_normal(D)).astype(np.float32)
    y = oracle.rmsnorm(x, None, 1e-6)
    yw = oracle.rmsnorm(x, w, 1e-6)
    assert np.array_equal(yw, (y * w).astype(np.float32))
    assert not np.allclose(yw, oracle.rmsnorm(x * w, None, 1e-6), rtol=1e-3)


# --------------------------------------------------------------------- RoPE

CS = workloads.cos_sin_cache(40000, D, 1e6)
CS64 = workloads.cos_sin_cache(40000, 64, 1e4)


@pytest.mark.parametrize("style,cs", [(0, CS), (1, CS), (1, CS64)])
def test_rope_position_zero_is_identity(style, cs):
    y = rng.standard_normal(D).astype(np.float32)
    assert np.array_equal(oracle.rope(y, cs[0], style)[: cs.shape[1]], y[: cs.shape[1]])


def _pairs(style, rot):
    half = rot // 2
    if style == 0:
        return np.arange(half), np.arange(half) + half
    return 2 * np.arange(half), 2 * np.arange(half) + 1


@pytest.mark.parametrize("style", [0, 1])
@pytest.mark.parametrize("pos", [1, 2, 17, 4095, 32767])
def test_rope_is_complex_multiplication(style, pos):
    """Each pair (a, b) maps to (a + ib)(cos + i sin); NeoX pairs i with
    i + rot/2, GPT-J pairs 2i with 2i + 1.  A wrong sign, pairing or cos/sin
    index fails this."""
    y = rng.standard_normal(D).astype(np.float32)
    row = CS[pos]
    o = oracle.rope(y, row, style).astype(np.float64)
    i0, i1 = _pairs(style, D)
    z = (y[i0].astype(np.float64) + 1j * y[i1].astype(np.float64)) * (
        row[: D // 2].astype(np.float64) + 1j * row[D // 2:].astype(np.float64))
    tol = 4e-7 * (np.abs(y[i0]) + np.abs(y[i1])) + 1e-30
    assert np.all(np.abs(o[i0] - z.real) <= tol)
    assert np.all(np.abs(o[i1] - z.imag) <= tol)


@pytest.mark.parametrize("style", [0, 1])
def test_rope_preserves_pair_norms(style):
    for pos in rng.integers(0, CS.shape[0], 50):
        y = (rng.standard_normal(D) * 3).astype(np.float32)
        o = oracle.rope(y, CS[pos], style).astype(np.float64)
        i0, i1 = _pairs(style, D)
        n_in = np.hypot(y[i0].astype(np.float64), y[i1].astype(np.float64))
        n_out = np.hypot(o[i0], o[i1])
        assert np.allclose(n_out, n_in, rtol=5e-7, atol=1e-30)


@pytest.mark.parametrize("style", [0, 1])
def test_rope_relative_position_invariance(style):
    """<R_m q, R_n k> depends only on m - n."""
    for _ in range(20):
        q = rng.standard_normal(D).astype(np.float32)
        k = rng.standard_normal(D).astype(np.float32)
        m, n, s = (int(v) for v in rng.integers(0, 12000, 3))
        d1 = np.dot(oracle.rope(q, CS[m], style).astype(np.float64),
                    oracle.rope(k, CS[n], style).astype(np.float64))
        d2 = np.dot(oracle.rope(q, CS[m + s], style).astype(np.float64),
                    oracle.rope(k, CS[n + s], style).astype(np.float64))
        # cos/sin rows are fp32 roundings of exact values: tolerance covers them
        assert abs(d1 - d2) <= 2e-5 * np.linalg.norm(q) * np.linalg.norm(k)


def test_rope_one_hot_neox():
    y = np.zeros(D, np.float32)
    y[5] = 1.0
    row = CS[123]
    o = oracle.rope(y, row, 0)
    assert o[5] == row[5] and o[5 + 64] == row[64 + 5]
    assert np.count_nonzero(o) == 2


def test_rope_gptj_partial_passes_rest_through():
    y = rng.standard_normal(D).astype(np.float32)
    o = oracle.rope(y, CS64[999], 1)
    assert np.array_equal(o[64:], y[64:])
    assert not np.array_equal(o[:64], y[:64])
