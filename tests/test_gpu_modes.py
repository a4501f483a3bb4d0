"""GPU parity of fqr_append_paged's optional modes against the oracle,
through the C ABI, under both schedules:

* the dynamic-Q prefill q_scale layout [B, Hq, round_up(max_seqlen, 128)]
  at the padding edges q_len 127 / 128 / 129, for (Hq, Hkv) (8, 1) and
  (64, 8), ragged batches with empty requests, the max_seqlen overflow flag
  (nothing written) and max_seqlen ignored outside policy 1;
* the Gemma-style norm x_hat * (1 + w) in every policy;
* caller-owned K/V rows (NULL caches and page table, every cache byte
  untouched, no page-overrun check);
* gate-tail rows [Q | K | V | G] (the G heads are never read)."""
import copy

import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from tests.gpu_harness import AppendRun

SCHEDULES = [1, 2]


def check(w, **kw):
    r = AppendRun(w, **kw)
    r.launch()
    rep = r.check()
    if not rep.get("flagged"):
        # the same correctly rounded steps on both sides: bit-identical
        assert rep.get("q_exact_frac", 1.0) == 1.0 and rep.get("k_exact_frac", 1.0) == 1.0, rep
        assert rep.get("q_scale_exact_frac", 1.0) == 1.0, rep
    return r, rep


# ------------------------------------------------------ prefill q_scale layout

@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("heads", [(8, 1), (64, 8)])
@pytest.mark.parametrize("q_len", [127, 128, 129])
def test_prefill_q_scale_padding_edges(q_len, heads, schedule):
    Hq, Hkv = heads
    w = workloads.make_append(seed=q_len + Hq, n_new=[q_len] * 4,
                              seq_lens=[q_len + 3, q_len, q_len + 64, q_len + 200],
                              Hq=Hq, Hkv=Hkv, page_size=64, max_pages=6, quant_policy=1,
                              norm_style=1, k_scale=0.05, v_scale=0.05, max_seqlen=q_len,
                              cos_sin_rows=512)
    r, rep = check(w, schedule=schedule)
    assert not rep.get("flagged")
    assert r.q_scale.shape == (4, Hq, -(-q_len // 128) * 128)


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("seed", [1, 2, 3])
def test_prefill_q_scale_ragged_with_empty_requests(seed, schedule):
    rng = np.random.default_rng(seed)
    n = rng.integers(0, 300, 9)
    n[[2, 5]] = 0
    L = n + rng.integers(0, 500, 9)
    w = workloads.make_append(seed=seed, n_new=n, seq_lens=L, Hq=16, Hkv=2, page_size=16,
                              max_pages=int(L.max()) // 16 + 1, quant_policy=1,
                              qkv_sigma=2.0, k_scale=0.05, v_scale=0.05,
                              max_seqlen=int(n.max()) + int(rng.integers(0, 200)),
                              cos_sin_rows=int(L.max()) + 1)
    _, rep = check(w, schedule=schedule)
    assert not rep.get("flagged")


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_max_seqlen_overflow_flags_all_and_writes_nothing(schedule):
    w = workloads.prefill_dynq_gemma(q_len=129)
    w.max_seqlen = 128                                   # every request has 129 rows
    r, rep = check(w, schedule=schedule)
    assert rep == {"flagged": True}
    assert (r.flags.cpu().numpy() == -1).all()


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("policy", [0, 2])
def test_max_seqlen_is_ignored_outside_dynamic_q(policy, schedule):
    w = workloads.make_append(seed=7, n_new=[40, 3], seq_lens=[50, 9], Hq=8, Hkv=2,
                              page_size=16, max_pages=4, quant_policy=policy,
                              q_scale_inv=20.0, k_scale=0.05, v_scale=0.05, max_seqlen=4)
    _, rep = check(w, schedule=schedule)
    assert not rep.get("flagged")


# --------------------------------------------------------------- Gemma norm

@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("policy", [0, 1, 2])
def test_gemma_norm(policy, schedule):
    rng = np.random.default_rng(policy)
    n = rng.integers(1, 60, 6)
    L = n + rng.integers(0, 100, 6)
    w = workloads.make_append(seed=30 + policy, n_new=n, seq_lens=L, Hq=32, Hkv=4,
                              page_size=16, max_pages=12, quant_policy=policy, qkv_sigma=2.0,
                              q_scale_inv=20.0, k_scale=0.05, v_scale=0.05, norm_style=1,
                              cos_sin_rows=200)
    _, rep = check(w, schedule=schedule)
    assert not rep.get("flagged")


# -------------------------------------------------------- caller-owned K / V

@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("policy", [0, 1, 2])
@pytest.mark.parametrize("null_caches", [True, False])
def test_owned_kv(policy, null_caches, schedule):
    rng = np.random.default_rng(40 + policy)
    n = rng.integers(0, 50, 7)
    L = n + rng.integers(0, 90, 7)
    w = workloads.make_append(seed=40 + policy, n_new=n, seq_lens=L, Hq=16, Hkv=4,
                              page_size=16, max_pages=10, quant_policy=policy, qkv_sigma=2.0,
                              q_scale_inv=20.0, k_scale=0.05, v_scale=0.05, out_kv=True,
                              cos_sin_rows=200)
    _, rep = check(w, schedule=schedule, null_caches=null_caches)
    assert not rep.get("flagged")


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_owned_kv_has_no_page_overrun_check(schedule):
    w = workloads.make_append(seed=50, n_new=[3, 5], seq_lens=[100, 70], Hq=8, Hkv=2,
                              page_size=16, max_pages=1, quant_policy=0, out_kv=True,
                              cos_sin_rows=128)           # 16 slots < 100
    _, rep = check(w, schedule=schedule, null_caches=False)
    assert not rep.get("flagged")
    paged = copy.copy(w)
    paged.out_kv = False
    _, rep = check(paged, schedule=schedule)
    assert rep == {"flagged": True}


# ---------------------------------------------------------------- gate tail

@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("policy", [0, 1, 2])
def test_gate_tail_rows(policy, schedule):
    rng = np.random.default_rng(60 + policy)
    n = rng.integers(0, 40, 5)
    L = n + rng.integers(0, 70, 5)
    w = workloads.make_append(seed=60 + policy, n_new=n, seq_lens=L, Hq=16, Hkv=2,
                              page_size=16, max_pages=8, quant_policy=policy,
                              q_scale_inv=20.0, k_scale=0.05, v_scale=0.05, gate_heads=16,
                              row_pad=8, cos_sin_rows=128)
    w.qkv[:, (16 + 4) * 128:] = 0x7FC0                   # NaN gates and padding
    _, rep = check(w, schedule=schedule)
    assert not rep.get("flagged")
