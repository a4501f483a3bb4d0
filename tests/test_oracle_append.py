"""Pins of the oracle's paged append (slots, tails, flags, validation, Q/K/V
quantisation) against an inverse-direction brute-force model and the
quantisation invariants.

The inverse model walks every cache row, asks which request owns its page and
which sequence position it holds, and from that alone decides whether the row
must hold a new token's K/V, zeros (past the end of the last page), or its old
bytes.  Expected K/V values come from the separately pinned step functions and
independent encoders (torch's BF16 conversion, a table-search E4M3)."""
import itertools
import math

import numpy as np
import pytest

import oracle
import workloads
from tests._util import bf16_bits_to_f32, bf16_rne_torch, e4m3_brute, e4m3_decode

D = 128


def run_oracle(w, fill_seed=1, **over):
    dt = np.uint16 if w.kv_esize == 2 else np.uint8
    rng = np.random.default_rng(fill_seed)
    shape = (w.num_pages, w.page_size, w.Hkv, D)
    hi = 1 << (8 * w.kv_esize)
    kc = rng.integers(0, hi, size=shape).astype(dt)
    vc = rng.integers(0, hi, size=shape).astype(dt)
    kc0, vc0 = kc.copy(), vc.copy()
    oq, qs, fl = oracle.new_outputs(w)
    rc = oracle.append_paged(w, kc, vc, oq, qs, fl, **over)
    return rc, (kc0, vc0), (kc, vc), (oq, qs, fl)


def post_rope(w, r, head, pos):
    """fp32 norm + rope of one head of packed row r (step functions)."""
    x = bf16_bits_to_f32(w.qkv[r, head * D:(head + 1) * D])
    wts = w.q_norm_w if head < w.Hq else w.k_norm_w
    y = oracle.rmsnorm(x, bf16_bits_to_f32(wts), w.eps) if wts is not None else x.copy()
    return oracle.rope(y, w.cos_sin[pos], w.rope_style)


def expected_kv(w, r, pos):
    """Expected K and V codes [Hkv, 128] of packed row r."""
    k = np.stack([post_rope(w, r, w.Hq + kh, pos) for kh in range(w.Hkv)])
    v_bits = np.stack([w.qkv[r, (w.Hq + w.Hkv + kh) * D:(w.Hq + w.Hkv + kh + 1) * D]
                       for kh in range(w.Hkv)])
    if w.quant_policy == 0:
        return bf16_rne_torch(k), v_bits
    ks, vs = np.float32(w.k_scale), np.float32(w.v_scale)
    return (e4m3_brute((k / ks).astype(np.float32)),
            e4m3_brute((bf16_bits_to_f32(v_bits) / vs).astype(np.float32)))


def check_inverse_model(w, before, after, page_table=None):
    pt = w.page_table if page_table is None else page_table
    P = w.page_size
    kc0, vc0 = before
    kc, vc = after
    n_new = np.diff(w.q_indptr)
    owner = {}
    for b in range(w.B):
        for k in range(math.ceil(int(w.seq_lens[b]) / P)):
            owner[int(pt[b, k])] = (b, k)
    for g in range(w.num_pages):
        for j in range(P):
            state = "old"
            if g in owner:
                b, k = owner[g]
                p, L, n = k * P + j, int(w.seq_lens[b]), int(n_new[b])
                if L - n <= p < L:
                    state = int(w.q_indptr[b]) + p - (L - n)  # the token stored here
                elif p >= L:
                    state = "zero"
            if state == "old":
                assert np.array_equal(kc[g, j], kc0[g, j]), (g, j)
                assert np.array_equal(vc[g, j], vc0[g, j]), (g, j)
            elif state == "zero":
                assert not kc[g, j].any() and not vc[g, j].any(), (g, j)
            else:
                r = state
                pos = int(w.positions[r]) if w.positions is not None else p
                ke, ve = expected_kv(w, r, pos)
                assert np.array_equal(kc[g, j], ke), (g, j, r)
                assert np.array_equal(vc[g, j], ve), (g, j, r)


def check_out_q(w, oq, qs):
    for b in range(w.B):
        lo, hi, L = int(w.q_indptr[b]), int(w.q_indptr[b + 1]), int(w.seq_lens[b])
        for r in range(lo, hi):
            pos = int(w.positions[r]) if w.positions is not None else r + L - hi
            o = np.stack([post_rope(w, r, h, pos) for h in range(w.Hq)])
            if w.quant_policy == 0:
                assert np.array_equal(oq[r], bf16_rne_torch(o))
            elif w.quant_policy == 2:
                assert np.array_equal(oq[r], e4m3_brute((o * np.float32(w.q_scale_inv)).astype(np.float32)))
            else:
                amax = np.abs(o).max(axis=1)
                want = (np.maximum(amax, np.float32(1e-6)) / np.float32(w.upper_max)).astype(np.float32)
                assert np.array_equal(qs[r], want)
                assert np.array_equal(oq[r], e4m3_brute((o / want[:, None]).astype(np.float32)))


def tiny(n_new, seq_lens, *, policy=0, seed=3, P=4, max_pages=3, Hq=2, Hkv=1, **kw):
    return workloads.make_append(
        seed=seed, n_new=n_new, seq_lens=seq_lens, Hq=Hq, Hkv=Hkv, page_size=P,
        max_pages=max_pages, quant_policy=policy, cos_sin_rows=max(12, max_pages * P),
        q_scale_inv=1 / 0.05, k_scale=0.05, v_scale=0.05, **kw)


# --------------------------------------------------------------- structure

@pytest.mark.parametrize("policy", [0, 2])
def test_inverse_model_one_request_every_length(policy):
    """B = 1, page 4, every (new tokens n, post-append length L) with L <= 12."""
    for L in range(0, 13):
        for n in range(0, L + 1):
            w = tiny([n], [L], policy=policy, seed=L * 13 + n)
            rc, before, after, (oq, qs, fl) = run_oracle(w)
            assert rc == 0 and list(fl) == [0]
            check_inverse_model(w, before, after)
            check_out_q(w, oq, qs)


@pytest.mark.parametrize("B", [2, 3])
def test_inverse_model_random_batches(B):
    rng = np.random.default_rng(B)
    for case in range(60):
        L = rng.integers(0, 13, B)
        n = np.array([rng.integers(0, l + 1) for l in L])
        w = tiny(n, L, policy=int(rng.integers(0, 3)), seed=100 + case, Hq=3, Hkv=2)
        rc, before, after, (oq, qs, fl) = run_oracle(w, fill_seed=case)
        assert rc == 0 and not fl.any()
        check_inverse_model(w, before, after)
        check_out_q(w, oq, qs)


def test_every_layout_of_a_six_page_table():
    w = tiny([3, 2], [7, 10], Hq=1, Hkv=1)
    for perm in itertools.permutations(range(6)):
        pt = np.array(perm, dtype=np.int32).reshape(2, 3)
        rc, before, after, _ = run_oracle(w, page_table=pt)
        assert rc == 0
        check_inverse_model(w, before, after, page_table=pt)


def test_explicit_positions_rotate_but_slots_follow_the_sequence():
    n, L = [3, 1], [9, 2]
    derived = np.array([6, 7, 8, 1])
    w = tiny(n, L, positions=derived + np.array([2, 0, 3, 5]), Hq=2, Hkv=2)
    rc, before, after, (oq, qs, fl) = run_oracle(w)
    assert rc == 0
    check_inverse_model(w, before, after)
    check_out_q(w, oq, qs)


# -------------------------------------------------------------- validation

def _valid_base(**kw):
    # requests: 2 new on length 5, empty on length 4, 3 new on length 3
    return tiny([2, 0, 3], [5, 4, 3], Hq=2, Hkv=1, **kw)


BAD_CASES = {
    "first_nonzero": dict(q_indptr=[1, 2, 2, 5]),
    "non_monotone": dict(q_indptr=[0, 3, 2, 5]),
    "last_short": dict(q_indptr=[0, 2, 2, 4]),
    "last_long": dict(q_indptr=[0, 2, 2, 6]),
    "seq_shorter_than_new": dict(seq_lens=[5, 4, 2]),
    "negative_seq_len": dict(seq_lens=[5, -1, 3]),
    "page_table_overrun": dict(seq_lens=[13, 4, 3]),
}


@pytest.mark.parametrize("case", sorted(BAD_CASES))
@pytest.mark.parametrize("policy", [0, 1, 2])
def test_each_malformed_predicate_flags_all_and_writes_nothing(case, policy):
    w = _valid_base(policy=policy)
    over = {k: np.array(v, dtype=np.int32) for k, v in BAD_CASES[case].items()}
    rc, (kc0, vc0), (kc, vc), (oq, qs, fl) = run_oracle(w, **over)
    oq0, qs0, _ = oracle.new_outputs(w)
    assert rc == 1 and list(fl) == [-1, -1, -1]
    assert np.array_equal(kc, kc0) and np.array_equal(vc, vc0)
    assert np.array_equal(oq, oq0) and np.array_equal(qs, qs0, equal_nan=True)


def test_cos_sin_row_overrun_is_flagged():
    w = tiny([1], [11], max_pages=3)
    w.cos_sin = w.cos_sin[:10]
    rc, before, after, (_, _, fl) = run_oracle(w)
    assert rc == 1 and list(fl) == [-1]
    assert np.array_equal(after[0], before[0])
    w.cos_sin = workloads.cos_sin_cache(11, D, 1e6)  # boundary: L == rows is valid
    assert run_oracle(w)[0] == 0


@pytest.mark.parametrize("bad_pos", [-1, 12])
def test_explicit_position_out_of_range_is_flagged(bad_pos):
    w = _valid_base(positions=[0, 1, 2, 3, bad_pos])
    rc, before, after, (_, _, fl) = run_oracle(w)
    assert rc == 1 and list(fl) == [-1] * 3
    assert np.array_equal(after[0], before[0]) and np.array_equal(after[1], before[1])


def test_boundaries_are_valid():
    # L == n (positions start at 0), L == max_pages * page_size
    w = tiny([3, 1], [3, 12])
    rc, before, after, (oq, qs, fl) = run_oracle(w)
    assert rc == 0 and not fl.any()
    check_inverse_model(w, before, after)


def test_empty_batch_and_requests_without_tokens():
    w = tiny([0, 0], [0, 6])
    rc, before, after, (_, _, fl) = run_oracle(w)
    assert rc == 0 and list(fl) == [0, 0]
    check_inverse_model(w, before, after)   # request 1 still gets its tail zeroed


# ------------------------------------------------------------ quantisation

@pytest.mark.parametrize("upper", [448.0, 240.0])
def test_dynamic_q_scale_invariants(upper):
    w = workloads.make_append(seed=11, n_new=[3, 1, 2], seq_lens=[40, 9, 100], Hq=4,
                              Hkv=2, page_size=16, max_pages=8, quant_policy=1,
                              qkv_sigma=2.0, k_scale=0.05, v_scale=0.05,
                              upper_max=upper)
    w.qkv[4, 2 * D:3 * D] = 0                    # one all-zero Q head
    rc, before, after, (oq, qs, fl) = run_oracle(w)
    assert rc == 0
    top = e4m3_brute(np.float32(upper))          # code of +upper_max
    for r in range(w.T):
        for h in range(w.Hq):
            vals = e4m3_decode(oq[r, h])
            if r == 4 and h == 2:
                assert qs[r, h] == np.float32(1e-6) / np.float32(upper)
                assert np.all(vals == 0)            # +-0 (rope of zeros gives -0 too)
                continue
            # the element at amax encodes to exactly +-upper_max
            assert np.abs(vals).max() == upper
            assert ((oq[r, h] & 0x7F) == top).any()
            b = int(np.searchsorted(w.q_indptr, r, side="right") - 1)
            pos = r + int(w.seq_lens[b]) - int(w.q_indptr[b + 1])
            o = post_rope(w, r, h, pos).astype(np.float64)
            assert qs[r, h] == pytest.approx(np.abs(o).max() / upper, rel=1e-6)
            # dequantised payload within E4M3 precision of the fp32 values
            err = np.abs(vals * qs[r, h] - o)
            assert np.all(err <= np.abs(o) * 2.0 ** -4 + qs[r, h] * 2.0 ** -10 + 1e-30)
    check_inverse_model(w, before, after)


def test_heads_with_very_different_scales_normalise_independently():
    """Adjacent heads scaled by 1e3 apart each come out with unit RMS (a
    reduction that mixed heads would fail)."""
    w = workloads.make_append(seed=5, n_new=[1, 1], seq_lens=[1, 1], Hq=8, Hkv=2,
                              page_size=4, max_pages=1, quant_policy=0)
    one = np.full(D, 0x3F80, np.uint16)
    w.q_norm_w, w.k_norm_w = one, one
    x = bf16_bits_to_f32(w.qkv).copy()
    for h in range(0, 12, 2):
        x[:, h * D:(h + 1) * D] *= 1e3
    w.qkv = (x.view(np.uint32) >> 16).astype(np.uint16)
    rc, _, (kc, vc), (oq, qs, fl) = run_oracle(w)
    assert rc == 0
    y = bf16_bits_to_f32(oq).astype(np.float64)          # position 0: no rotation
    assert np.allclose(np.sqrt((y ** 2).mean(axis=2)), 1.0, rtol=1e-2)
