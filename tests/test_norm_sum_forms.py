"""Host emulation of the two ways the kernels form the exact mean square of a
head (fqr_head.cuh, inv_rms_n: kSumMixed and kSumShort), in the kernels' own
summation order, against the oracle's RMSNorm of the same heads.

This pins, on the host, the bit identities and range bounds those forms rely
on:
- kSumMixed: the binary64 high word ((u & 0x7FFF0000) >> 3) + (896 << 20) of a
  BF16 value's fp32 bits u is |x| for every finite normal value, and the rare
  NaN branch;
- kSumShort: a non-negative binary32 square p shifted right by 3 is the high
  word of p * 2^-896 for exact squares, the sum's scaling by 2^889, and the
  [2^-60, 2^121) range outside which the general path runs.
The kernels themselves are compared with the oracle on the GPU
(tests/test_gpu_append.py); this emulation shares no code with them.
"""
import numpy as np
import pytest

import oracle

D = 128


def _lane_pairs(x):
    """The 8 lanes' 8 (first, second) pairs of a head, as the kernels hold them:
    lane l owns elements [8l, 8l + 8) and [64 + 8l, 64 + 8l + 8)."""
    out = []
    for l8 in range(8):
        idx = list(range(8 * l8, 8 * l8 + 8)) + list(range(64 + 8 * l8, 64 + 8 * l8 + 8))
        v = x[idx]
        out.append([(v[2 * j], v[2 * j + 1]) for j in range(8)])
    return out


def _hi_word_double(hi):
    return np.array([np.uint64(int(hi) & 0xFFFFFFFF) << np.uint64(32)]).view(np.float64)[0]


def _xor_tree(lane_sums):
    s = list(lane_sums)
    for m in (4, 2, 1):
        s = [s[i] + s[i ^ m] for i in range(8)]
    assert all(v == s[0] or (np.isnan(v) and np.isnan(s[0])) for v in s)
    return s[0]


def _general(x):
    ss = 0.0
    for v in x.astype(np.float64):
        ss = ss + v * v
    return np.float32(ss * (1.0 / D))


def mean_square_mixed(x):
    lanes = []
    for pairs in _lane_pairs(x):
        s = [0.0, 0.0, 0.0, 0.0]
        for j, (a, b) in enumerate(pairs):
            u = np.float64(a)
            ub = int(np.array([b], np.float32).view(np.uint32)[0])
            v = _hi_word_double(((ub & 0x7FFF0000) >> 3) + 0x38000000)
            s[(j & 1) * 2] = s[(j & 1) * 2] + u * u        # an exact product: one rounding, as an FMA
            s[(j & 1) * 2 + 1] = s[(j & 1) * 2 + 1] + v * v
        lanes.append((s[0] + s[1]) + (s[2] + s[3]))
    with np.errstate(over="ignore", invalid="ignore"):
        ms = np.float32(_xor_tree(lanes) * (1.0 / D))
    if ms == np.inf and np.isnan(x).any():
        ms = np.float32(np.nan)
    return ms


def mean_square_short(x):
    lanes = []
    for pairs in _lane_pairs(x):
        s = [0.0, 0.0, 0.0, 0.0]
        for j, (a, b) in enumerate(pairs):
            with np.errstate(over="ignore", under="ignore", invalid="ignore"):
                p = np.array([a, b], np.float32) * np.array([a, b], np.float32)
            bits = p.view(np.uint32)
            s[(j & 1) * 2] = s[(j & 1) * 2] + _hi_word_double(int(bits[0]) >> 3)
            s[(j & 1) * 2 + 1] = s[(j & 1) * 2 + 1] + _hi_word_double(int(bits[1]) >> 3)
        lanes.append((s[0] + s[1]) + (s[2] + s[3]))
    with np.errstate(over="ignore"):
        ms = np.float32(_xor_tree(lanes) * 2.0 ** 889)
    if not (2.0 ** -60 <= ms < 2.0 ** 121):
        with np.errstate(over="ignore", invalid="ignore"):
            ms = _general(x)
    return ms


def normed(x, w, eps, mean_square):
    """(x * inv) * w with inv = RN(1 / RN(sqrt(RN(ms + eps)))) in fp32."""
    with np.errstate(all="ignore"):
        v = np.float32(mean_square(x)) + np.float32(eps)
        inv = np.float32(1.0) / np.sqrt(np.float32(v))
        return (x * inv).astype(np.float32) * w


def _bf16(a):
    return oracle.bf16_to_f32(oracle.bf16(np.asarray(a, np.float32)))


def _bits(b):
    """The fp32 value of one BF16 bit pattern."""
    return oracle.bf16_to_f32(np.array([b], np.uint16))[0]


def _heads():
    rng = np.random.default_rng(2024)
    heads = []
    for k in range(120):   # N(0, 1) heads over a wide range of scales
        heads.append(_bf16(rng.standard_normal(D) * 2.0 ** rng.integers(-55, 60)))
    for k in range(20):    # zeros among them
        h = _bf16(rng.standard_normal(D))
        h[rng.integers(0, D, 40)] = 0.0
        heads.append(h)
    bits = rng.integers(0, 1 << 16, D).astype(np.uint16)
    special = [
        lambda h: h.__setitem__(5, np.nan),
        lambda h: h.__setitem__(6, np.nan),
        lambda h: h.__setitem__(3, np.inf),
        lambda h: h.__setitem__(100, -np.inf),
        lambda h: h.__setitem__(slice(None), oracle.bf16_to_f32(np.full(D, 0x7F7F, np.uint16))),
        lambda h: h.__setitem__(slice(None), oracle.bf16_to_f32(rng.integers(1, 0x80, D).astype(np.uint16))),
        lambda h: h.__setitem__(slice(None), 0.0),
        lambda h: (h.__setitem__(slice(None), 0.0), h.__setitem__(77, 1.0)),
        lambda h: h.__setitem__(slice(None), oracle.bf16_to_f32(bits & 0x80FF | 0x0080)),
        lambda h: h.__setitem__(slice(None), oracle.bf16_to_f32(bits & 0x807F | 0x3080)),
        lambda h: h.__setitem__(slice(None), np.where(rng.random(D) < 0.5, h, _bits(0x1CC1))),
        lambda h: h.__setitem__(40, _bits(0x5F35)),
        lambda h: h.__setitem__(41, _bits(0x6780)),
    ]
    for fn in special:
        h = _bf16(rng.standard_normal(D))
        fn(h)
        heads.append(h.astype(np.float32))
    return heads


@pytest.mark.parametrize("form", ["mixed", "short"])
def test_sum_forms_match_the_oracle_bitwise(form):
    ms = mean_square_mixed if form == "mixed" else mean_square_short
    rng = np.random.default_rng(7)
    w = _bf16(1.0 + 0.25 * rng.standard_normal(D))
    for i, x in enumerate(_heads()):
        got = normed(x, w, 1e-6, ms)
        want = oracle.rmsnorm(x, w, 1e-6)
        same = (got.view(np.uint32) == want.view(np.uint32)) | (np.isnan(got) & np.isnan(want))
        assert same.all(), (form, i, np.flatnonzero(~same)[:4])


def test_bit_identities_of_the_conversions():
    """Every finite normal BF16 value: the mixed form's high word is |x|; every
    square of such a value inside [2^-63, 2^64): the short form's shift is the
    square times 2^-896."""
    b = np.arange(1 << 16, dtype=np.uint32)
    e = (b >> 7) & 0xFF
    with np.errstate(invalid="ignore"):
        x = oracle.bf16_to_f32(b.astype(np.uint16)).astype(np.float64)
    u = b << 16
    hi = (((u & 0x7FFF0000) >> 3) + 0x38000000).astype(np.uint64) << np.uint64(32)
    normal = (e > 0) & (e < 0xFF)
    assert (hi.view(np.float64)[normal] == np.abs(x[normal])).all()
    inside = normal & (np.abs(x) >= 2.0 ** -63) & (np.abs(x) < 2.0 ** 64)
    p = (x[inside] * x[inside]).astype(np.float32)
    assert (p.astype(np.float64) == x[inside] ** 2).all()          # the fp32 squares are exact
    pb = p.view(np.uint32)
    assert ((pb & 7) == 0).all()                                     # so the low word is zero
    d = ((pb >> 3).astype(np.uint64) << np.uint64(32)).view(np.float64)
    assert (d == p.astype(np.float64) * 2.0 ** -896).all()
