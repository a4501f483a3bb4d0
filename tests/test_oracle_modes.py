"""Pins of the oracle's optional modes against the pinned base path.

* prefill q_scale layout [B, Hq, round_up(max_seqlen, 128)], addressed by the
  token's index inside its request (FlashInfer PR #5956, "Contract"), with the
  n_b <= max_seqlen check ("max_seqlen overflow -> all flags -1");
* the Gemma-style norm, x_hat * (1 + w) (TensorRT-LLM PR #16024,
  "qk_norm_use_gemma"): special weights that reduce it to known cases, and a
  one-hot closed form;
* caller-owned K/V outputs (FlashInfer PR #5956 review: redirected K/V writes
  leave the paged caches alone);
* gate-tail rows [Q | K | V | G] (TensorRT-LLM PR #16024, "Gate-tail QKV
  layout"): the G heads never change a result."""
import copy

import numpy as np
import pytest

import oracle
import workloads
from tests._util import bf16_bits_to_f32, bf16_rne_torch
from tests.test_oracle_append import run_oracle

D = 128


def dynq(n_new, seq_lens, max_seqlen, *, seed=21, Hq=4, Hkv=2, P=16, **kw):
    return workloads.make_append(
        seed=seed, n_new=n_new, seq_lens=seq_lens, Hq=Hq, Hkv=Hkv, page_size=P,
        max_pages=-(-max(seq_lens) // P), quant_policy=1, k_scale=0.05, v_scale=0.05,
        max_seqlen=max_seqlen, **kw)


# ------------------------------------------------------ prefill q_scale layout

@pytest.mark.parametrize("q_len", [127, 128, 129])
def test_prefill_layout_holds_the_decode_scales_by_index_in_request(q_len):
    n = [q_len, 0, q_len - 5, 1]
    L = [q_len + 7, 3, q_len, 40]
    wp = dynq(n, L, q_len)
    wd = copy.copy(wp)
    wd.max_seqlen = 0
    rp, before, after_p, (oq_p, qs_p, fl_p) = run_oracle(wp)
    rd, _, after_d, (oq_d, qs_d, fl_d) = run_oracle(wd)
    assert rp == 0 and rd == 0 and not fl_p.any()
    ld = -(-q_len // 128) * 128
    assert qs_p.shape == (4, wp.Hq, ld)
    want = np.full(qs_p.shape, np.nan, np.float32)
    for b in range(wp.B):
        lo, hi = int(wp.q_indptr[b]), int(wp.q_indptr[b + 1])
        want[b, :, : hi - lo] = qs_d[lo:hi].T         # token index inside the request
    assert np.array_equal(qs_p, want, equal_nan=True)  # padding entries untouched
    assert np.array_equal(oq_p, oq_d)
    assert all(np.array_equal(a, b) for a, b in zip(after_p, after_d))


def test_max_seqlen_overflow_flags_everything_and_writes_nothing():
    w = dynq([5, 3], [9, 20], 4)                       # request 0 has 5 > 4 rows
    rc, (kc0, vc0), (kc, vc), (oq, qs, fl) = run_oracle(w)
    oq0, qs0, _ = oracle.new_outputs(w)
    assert rc == 1 and list(fl) == [-1, -1]
    assert np.array_equal(kc, kc0) and np.array_equal(vc, vc0)
    assert np.array_equal(oq, oq0) and np.array_equal(qs, qs0, equal_nan=True)
    w.max_seqlen = 5                                    # boundary: n_b == max_seqlen
    assert run_oracle(w)[0] == 0


@pytest.mark.parametrize("policy", [0, 2])
def test_max_seqlen_is_a_dynamic_q_prefill_argument_only(policy):
    w = workloads.make_append(seed=4, n_new=[5, 3], seq_lens=[9, 20], Hq=2, Hkv=1,
                              page_size=16, max_pages=2, quant_policy=policy,
                              q_scale_inv=20.0, k_scale=0.05, v_scale=0.05, max_seqlen=4)
    assert oracle.validate(w.q_indptr, w.seq_lens, w.T, w.max_pages, 16, w.cos_sin_rows,
                           max_seqlen=4) == 1
    assert run_oracle(w)[0] == 0


# ------------------------------------------------------------- Gemma norm

def _gemma_pair(wbits, policy=0, seed=8):
    base = workloads.make_append(seed=seed, n_new=[2, 1], seq_lens=[5, 30], Hq=4, Hkv=2,
                                 page_size=16, max_pages=2, quant_policy=policy,
                                 q_scale_inv=20.0, k_scale=0.05, v_scale=0.05)
    g = copy.copy(base)
    g.norm_style = 1
    g.q_norm_w = np.full(D, wbits, np.uint16)
    g.k_norm_w = np.full(D, wbits, np.uint16)
    return base, g


@pytest.mark.parametrize("policy", [0, 1, 2])
def test_gemma_with_zero_weights_is_the_unit_weight_norm(policy):
    base, g = _gemma_pair(0x0000, policy)
    base.q_norm_w = np.full(D, 0x3F80, np.uint16)      # 1.0
    base.k_norm_w = np.full(D, 0x3F80, np.uint16)
    rb, _, after_b, out_b = run_oracle(base)
    rg, _, after_g, out_g = run_oracle(g)
    assert rb == rg == 0
    assert all(np.array_equal(x, y, equal_nan=True) for x, y in zip(after_b + out_b, after_g + out_g))


def test_gemma_with_minus_one_weights_zeroes_q_and_k():
    _, g = _gemma_pair(0xBF80)                          # -1.0: 1 + w = 0
    rc, _, (kc, vc), (oq, qs, fl) = run_oracle(g)
    assert rc == 0
    assert np.all((oq & 0x7FFF) == 0)                   # +-0 in BF16
    # the K slots of the three tokens hold +-0 as well
    P = g.page_size
    for b in range(g.B):
        lo, hi, L = int(g.q_indptr[b]), int(g.q_indptr[b + 1]), int(g.seq_lens[b])
        for r in range(lo, hi):
            p = r + L - hi
            assert np.all((kc[g.page_table[b, p // P], p % P] & 0x7FFF) == 0)


def test_gemma_one_hot_closed_form():
    """x = a e_k at position 0 (no rotation): y_k = a / sqrt(a^2/128 + eps) * (1 + w_k)."""
    w = workloads.make_append(seed=9, n_new=[1], seq_lens=[1], Hq=2, Hkv=1, page_size=4,
                              max_pages=1, quant_policy=0, norm_style=1)
    rng = np.random.default_rng(3)
    for trial in range(40):
        k = int(rng.integers(0, D))
        a = np.float32(rng.choice([-1, 1]) * 2.0 ** rng.uniform(-6, 6))
        x = np.zeros(w.row_stride, np.float32)
        x[k] = a
        w.qkv = (x.view(np.uint32) >> 16).astype(np.uint16)[None, :]
        a = bf16_bits_to_f32(w.qkv[0, k])
        rc, _, _, (oq, _, _) = run_oracle(w)
        assert rc == 0
        wk = np.float64(bf16_bits_to_f32(w.q_norm_w[k]))
        want = np.float64(a) / np.sqrt(np.float64(a) ** 2 / 128 + 1e-6) * (1.0 + wk)
        got = bf16_bits_to_f32(oq[0, 0]).astype(np.float64)
        assert abs(got[k] - want) <= abs(want) * 2.0 ** -8 + 1e-30
        assert not np.delete(got, k).any()


def test_gemma_differs_from_the_plain_norm():
    base = workloads.make_append(seed=12, n_new=[1], seq_lens=[3], Hq=2, Hkv=1,
                                 page_size=4, max_pages=1, quant_policy=0)
    g = copy.copy(base)
    g.norm_style = 1
    assert not np.array_equal(run_oracle(base)[3][0], run_oracle(g)[3][0])


# ------------------------------------------------------ caller-owned K / V

def _paged_and_owned(policy, seed=13):
    w = workloads.make_append(seed=seed, n_new=[3, 0, 2], seq_lens=[7, 5, 18], Hq=4, Hkv=2,
                              page_size=4, max_pages=5, quant_policy=policy,
                              q_scale_inv=20.0, k_scale=0.05, v_scale=0.05)
    o = copy.copy(w)
    o.out_kv = True
    return w, o


@pytest.mark.parametrize("policy", [0, 1, 2])
def test_owned_kv_rows_equal_the_cache_slots_and_the_caches_stay(policy):
    w, o = _paged_and_owned(policy)
    rc, _, (kc, vc), out_w = run_oracle(w)
    ok, ov = oracle.new_kv_outputs(o)
    rc2, (kc0, vc0), (kc2, vc2), out_o = run_oracle(o, out_k=ok, out_v=ov)
    assert rc == rc2 == 0
    assert np.array_equal(kc2, kc0) and np.array_equal(vc2, vc0)   # no slot, no tail
    assert all(np.array_equal(x, y, equal_nan=True) for x, y in zip(out_w, out_o))
    P = w.page_size
    for b in range(w.B):
        lo, hi, L = int(w.q_indptr[b]), int(w.q_indptr[b + 1]), int(w.seq_lens[b])
        for r in range(lo, hi):
            p = r + L - hi
            pg = w.page_table[b, p // P]
            assert np.array_equal(ok[r], kc[pg, p % P]) and np.array_equal(ov[r], vc[pg, p % P])


def test_owned_kv_skips_the_page_overrun_check():
    w, o = _paged_and_owned(0)
    short = np.ascontiguousarray(w.page_table[:, :2])  # 8 slots < 18
    assert run_oracle(w, page_table=short)[0] == 1
    ok, ov = oracle.new_kv_outputs(o)
    assert run_oracle(o, page_table=short, out_k=ok, out_v=ov)[0] == 0


# ------------------------------------------------------------ gate tail

@pytest.mark.parametrize("policy", [0, 1, 2])
def test_gate_heads_change_nothing(policy):
    kw = dict(seed=14, n_new=[2, 3], seq_lens=[6, 9], Hq=4, Hkv=2, page_size=4,
              max_pages=3, quant_policy=policy, q_scale_inv=20.0, k_scale=0.05,
              v_scale=0.05)
    g = workloads.make_append(gate_heads=4, **kw)
    H = (4 + 2 * 2) * D
    p = copy.copy(g)                                     # the same rows without G
    p.qkv = np.ascontiguousarray(g.qkv[:, :H])
    p.row_stride, p.gate_heads = H, 0
    res = [run_oracle(x) for x in (g, p)]
    g2 = copy.copy(g)
    g2.qkv = g.qkv.copy()
    g2.qkv[:, H:] = 0x7FC0                               # NaN gates
    res.append(run_oracle(g2))
    for r in res[1:]:
        assert r[0] == res[0][0] == 0
        assert all(np.array_equal(x, y, equal_nan=True)
                   for x, y in zip(r[2] + r[3], res[0][2] + res[0][3]))
