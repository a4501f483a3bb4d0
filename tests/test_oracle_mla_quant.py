"""Pins of the oracle's MLA Q quantisation (vLLM issue #24678: static
per-tensor, dynamic per-token and dynamic per-group scales for Q; the
scale/payload form of the dynamic per-head Q scale of FlashInfer PR #5956,
"Contract").

The values v = [nope | rope(rope part)] come from the separately pinned step
functions; the checks are the invariants the definitions fix: the element at
the token's (head's) maximum encodes to +-upper_max, dequantised payloads
stay within E4M3 precision, the per-token scale is the largest per-head
scale, the nope part of a static scale of 1 is the E4M3 code of its BF16
input, Q and the latent rows are what the unquantised call leaves."""
import copy

import numpy as np
import pytest

import oracle
import workloads
from tests._util import bf16_bits_to_f32, e4m3_brute, e4m3_decode
from tests.test_oracle_mla import run


def small(q_quant, seed=3, upper=448.0, qsi=1 / 0.02):
    n = [2, 1, 3]
    return workloads.make_mla(seed=seed, n_new=n, seq_lens=[9, 1, 70], Hq=6, block_size=16,
                              max_blocks=5, q_quant=q_quant, q_scale_inv=qsi, upper_max=upper)


def run_q(w):
    q_out, q_scale = oracle.new_mla_q_outputs(w)
    rc, q, lat0, lat, flags = run(w, q_out=q_out, q_scale=q_scale)
    return rc, q, lat, flags, q_out, q_scale


def values(w, r):
    b = int(np.searchsorted(w.q_indptr, r, side="right") - 1)
    pos = r + int(w.seq_lens[b]) - int(w.q_indptr[b + 1])
    v = bf16_bits_to_f32(w.q[r]).copy()
    for h in range(w.Hq):
        v[h, w.nope_dim:] = oracle.rope(v[h, w.nope_dim:], w.cos_sin[pos], w.rope_style)
    return v.astype(np.float64)


@pytest.mark.parametrize("q_quant", [1, 2, 3])
def test_q_is_read_only_and_latent_rows_match_the_unquantised_call(q_quant):
    w = small(q_quant)
    rc, q, lat, flags, _, _ = run_q(w)
    base = copy.copy(w)
    base.q_quant = 0
    rc0, _, _, lat_base, _ = run(base)
    assert rc == rc0 == 0 and not flags.any()
    assert np.array_equal(q, w.q)
    assert np.array_equal(lat, lat_base)


@pytest.mark.parametrize("upper", [448.0, 240.0])
@pytest.mark.parametrize("q_quant", [2, 3])
def test_dynamic_scale_invariants(q_quant, upper):
    w = small(q_quant, upper=upper)
    rc, _, _, _, q_out, q_scale = run_q(w)
    assert rc == 0
    top = e4m3_brute(np.float32(upper))
    for r in range(w.T):
        v = values(w, r)
        dec = e4m3_decode(q_out[r])
        groups = [(slice(None), r)] if q_quant == 2 else [(h, (r, h)) for h in range(w.Hq)]
        for sel, idx in groups:
            s = float(q_scale[idx])
            assert s == pytest.approx(np.abs(v[sel]).max() / upper, rel=1e-6)
            assert np.abs(dec[sel]).max() == upper
            assert ((q_out[r][sel] & 0x7F) == top).any()
            err = np.abs(dec[sel] * s - v[sel])
            assert np.all(err <= np.abs(v[sel]) * 2.0 ** -4 + s * 2.0 ** -10 + 1e-30)


def test_per_token_scale_is_the_largest_per_head_scale():
    wt, wh = small(2), small(3)
    qt, qh = run_q(wt)[5], run_q(wh)[5]
    assert np.array_equal(qt, qh.max(axis=1))


def test_static_unit_scale_nope_part_is_the_e4m3_code_of_the_input():
    w = small(1, qsi=1.0)
    rc, _, _, _, q_out, _ = run_q(w)
    assert rc == 0
    nope = bf16_bits_to_f32(w.q[:, :, :w.nope_dim])
    assert np.array_equal(q_out[:, :, :w.nope_dim], e4m3_brute(nope))


def test_static_scale_dequantises_within_e4m3_precision():
    w = small(1)
    rc, _, _, _, q_out, _ = run_q(w)
    qsi = np.float64(np.float32(w.q_scale_inv))
    for r in range(w.T):
        v = values(w, r) * qsi
        dec = e4m3_decode(q_out[r])
        sat = np.abs(v) >= 464
        assert np.all(np.abs(dec[~sat] - v[~sat]) <= np.abs(v[~sat]) * 2.0 ** -4 + 2.0 ** -10)
        assert np.all(np.abs(dec[sat]) == 448)


@pytest.mark.parametrize("q_quant", [2, 3])
def test_all_zero_token(q_quant):
    w = small(q_quant)
    w.q[1] = 0
    rc, _, _, _, q_out, q_scale = run_q(w)
    assert rc == 0
    assert np.all(e4m3_decode(q_out[1]) == 0)
    want = np.float32(1e-6) / np.float32(w.upper_max)
    assert np.all(q_scale[1] == want)


def test_flagged_call_writes_no_q_output():
    w = small(3)
    q_out, q_scale = oracle.new_mla_q_outputs(w)
    q0, s0 = q_out.copy(), q_scale.copy()
    rc, *_ = run(w, q_out=q_out, q_scale=q_scale, q_indptr=np.array([0, 2, 1, 6], np.int32))
    assert rc == 1
    assert np.array_equal(q_out, q0) and np.array_equal(q_scale, s0, equal_nan=True)


# ---------------------------------------------------------- per-group scales

def small_group(G, seed=3, upper=448.0):
    w = small(4, seed=seed, upper=upper)
    w.q_group = G
    return w


@pytest.mark.parametrize("upper", [448.0, 240.0])
@pytest.mark.parametrize("G", [8, 64, 128, 192])
def test_group_scale_invariants(G, upper):
    """Each group of G consecutive values of a head (the last one shorter when
    G does not divide the head width) has s = max|v| / upper_max, holds a code
    of exactly +-upper_max at its maximum, and dequantises within E4M3
    precision."""
    w = small_group(G, upper=upper)
    rc, _, _, _, q_out, q_scale = run_q(w)
    assert rc == 0
    W = w.nope_dim + w.rope_dim
    ng = -(-W // G)
    assert q_scale.shape == (w.T, w.Hq, ng)
    top = e4m3_brute(np.float32(upper))
    for r in range(w.T):
        v = values(w, r)
        dec = e4m3_decode(q_out[r])
        for h in range(w.Hq):
            for k in range(ng):
                sl = slice(k * G, min(W, (k + 1) * G))
                s = float(q_scale[r, h, k])
                assert s == pytest.approx(np.abs(v[h, sl]).max() / upper, rel=1e-6)
                assert np.abs(dec[h, sl]).max() == upper
                assert ((q_out[r, h, sl] & 0x7F) == top).any()
                err = np.abs(dec[h, sl] * s - v[h, sl])
                assert np.all(err <= np.abs(v[h, sl]) * 2.0 ** -4 + s * 2.0 ** -10 + 1e-30)


@pytest.mark.parametrize("G", [192, 256, 1000])
def test_group_as_wide_as_the_head_is_the_per_head_scale(G):
    """G >= nope + rope: one group per head, bit for bit the per-head mode."""
    wg, wh = small_group(G), small(3)
    _, _, _, _, qg, sg = run_q(wg)
    _, _, _, _, qh, sh = run_q(wh)
    assert np.array_equal(qg, qh)
    assert np.array_equal(sg[..., 0], sh)


def test_group_of_128_splits_nope_and_rope():
    """With nope 128 and rope 64, G = 128 gives two groups per head: the nope
    part (raw BF16 values) and the rotated rope part."""
    w = small_group(128)
    rc, _, _, _, q_out, q_scale = run_q(w)
    for r in range(w.T):
        v = values(w, r)
        assert np.allclose(q_scale[r, :, 0], np.abs(v[:, :128]).max(axis=1) / w.upper_max,
                           rtol=1e-6)
        assert np.allclose(q_scale[r, :, 1], np.abs(v[:, 128:]).max(axis=1) / w.upper_max,
                           rtol=1e-6)


def test_all_zero_group():
    """A group whose values are all zero gets the floor scale 1e-6 / upper_max
    and zero codes; the head's other groups are unaffected."""
    w = small_group(64)
    w.q[1, 2, :64] = 0          # the first group of head 2 of row 1
    rc, _, _, _, q_out, q_scale = run_q(w)
    assert rc == 0
    assert q_scale[1, 2, 0] == np.float32(1e-6) / np.float32(w.upper_max)
    assert np.all(e4m3_decode(q_out[1, 2, :64]) == 0)
    assert q_scale[1, 2, 1] > 1e-4 and np.abs(e4m3_decode(q_out[1, 2, 64:])).max() == w.upper_max
