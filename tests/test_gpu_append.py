"""GPU parity of fqr_append_paged against the oracle, through the C ABI.

Full-size named workloads (in the launch configuration bench.py times), the
malformed-metadata run, and a sweep of small ragged cases spanning several
tiles and ragged tails, plus edge cases: requests without tokens, every
malformed predicate, the largest batch, padded rows and page strides,
explicit positions, norm off, all 65536 BF16 inputs through the FP8 encoder,
the reduction-scope guard, a non-default stream and CUDA-graph replay."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._util import bf16_bits_to_f32, ulp_e4m3

pytestmark = pytest.mark.gpu
D = 128

if torch.cuda.is_available():
    from tests.gpu_harness import AppendRun, _np


SCHEDULES = [1, 2]   # latency, streaming: every case runs under both


def run_and_check(w, **kw):
    r = AppendRun(w, **kw)
    r.launch()
    rep = r.check()
    return r, rep


@pytest.mark.parametrize("schedule", [0] + SCHEDULES)
@pytest.mark.parametrize("name", sorted(workloads.APPEND_CONFIGS))
def test_named_workload_parity(name, schedule):
    w = workloads.APPEND_CONFIGS[name]()
    _, rep = run_and_check(w, schedule=schedule)
    print(name, schedule, rep)
    assert not rep.get("flagged")
    # the kernel and the oracle take the same correctly rounded steps (the
    # mean square as the rounded exact mean, every product rounded): beyond
    # the <= 1 ulp bar, the named workloads come out bit-identical
    assert rep["q_exact_frac"] == 1.0 and rep.get("k_exact_frac", 1.0) == 1.0, rep
    assert rep.get("q_scale_exact_frac", 1.0) == 1.0, rep


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_ragged_prefill_malformed_indptr_writes_nothing(schedule):
    w = workloads.ragged_prefill_fp8()
    r = AppendRun(w, q_indptr=workloads.malformed_indptr(w), schedule=schedule)
    r.launch()
    rep = r.check()
    assert rep == {"flagged": True}
    assert (r.flags.cpu().numpy() == -1).all()


SWEEP = [
    # (P, Hq, Hkv, policy, style, rot, norm, positions, row_pad)
    (4, 8, 1, 0, 0, 128, True, False, 0),
    (16, 32, 8, 0, 0, 128, True, False, 64),
    (64, 64, 8, 1, 0, 128, True, False, 0),
    (16, 64, 8, 2, 0, 128, True, False, 0),
    (128, 8, 1, 1, 0, 128, True, True, 0),
    (16, 4, 4, 2, 1, 128, True, False, 8),
    (64, 16, 2, 1, 1, 64, True, False, 0),
    (16, 6, 2, 0, 1, 2, False, False, 0),
    (32, 12, 4, 2, 0, 128, False, True, 0),
    (1, 8, 8, 1, 0, 128, True, False, 0),
    (16, 128, 8, 1, 0, 128, True, False, 0),
]


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("P,Hq,Hkv,policy,style,rot,norm,pos,pad", SWEEP)
@pytest.mark.parametrize("seed", [1, 2])
def test_small_ragged_sweep(P, Hq, Hkv, policy, style, rot, norm, pos, pad, seed, schedule):
    rng = np.random.default_rng(seed * 1000 + P + Hq)
    B = 7
    n = rng.integers(0, 40, B)
    n[rng.integers(0, B)] = 0
    prior = rng.integers(0, 3 * P + 5, B)
    L = prior + n
    max_pages = int(np.ceil(L.max() / P)) + 1
    rows = int(L.max()) + 7
    positions = None
    if pos:
        positions = rng.integers(0, rows, int(n.sum()))
    w = workloads.make_append(seed=seed, n_new=n, seq_lens=L, Hq=Hq, Hkv=Hkv, page_size=P,
                              max_pages=max_pages, num_pages=B * max_pages + 3,
                              quant_policy=policy, qkv_sigma=2.0, norm=norm, rot_dim=rot,
                              rope_style=style, cos_sin_rows=rows, row_pad=pad,
                              positions=positions, q_scale_inv=1 / 0.05, k_scale=0.05,
                              v_scale=0.05)
    _, rep = run_and_check(w, schedule=schedule)
    # both sides evaluate the same correctly rounded steps: bit-identical
    assert rep["q_exact_frac"] == 1.0 and rep.get("k_exact_frac", 1.0) == 1.0, rep


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_requests_without_tokens_only_tails_and_flags(schedule):
    w = workloads.make_append(seed=3, n_new=[0, 0, 0, 0], seq_lens=[0, 5, 16, 33], Hq=8, Hkv=2,
                              page_size=16, max_pages=3, quant_policy=1, cos_sin_rows=40,
                              k_scale=0.05, v_scale=0.05)
    r, _ = run_and_check(w, schedule=schedule)
    assert (r.flags.cpu().numpy() == 0).all()


BAD = {
    "first_nonzero": dict(q_indptr=[1, 2, 2, 5]),
    "non_monotone": dict(q_indptr=[0, 3, 2, 5]),
    "last_short": dict(q_indptr=[0, 2, 2, 4]),
    "last_long": dict(q_indptr=[0, 2, 2, 6]),
    "seq_shorter_than_new": dict(seq_lens=[5, 4, 2]),
    "negative_seq_len": dict(seq_lens=[5, -1, 3]),
    "page_table_overrun": dict(seq_lens=[13, 4, 3]),
    "cos_sin_overrun": dict(seq_lens=[5, 4, 12]),
}


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("case", sorted(BAD))
@pytest.mark.parametrize("policy", [0, 1, 2])
def test_each_malformed_predicate_writes_nothing(case, policy, schedule):
    w = workloads.make_append(seed=4, n_new=[2, 0, 3], seq_lens=[5, 4, 3], Hq=4, Hkv=2,
                              page_size=4, max_pages=3, quant_policy=policy, cos_sin_rows=11,
                              k_scale=0.05, v_scale=0.05, q_scale_inv=20.0)
    over = {k: np.array(v, np.int32) for k, v in BAD[case].items()}
    r = AppendRun(w, schedule=schedule, **over)
    r.launch()
    assert r.check() == {"flagged": True}
    assert (r.flags.cpu().numpy() == -1).all()


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("bad", [-1, 11])
def test_explicit_position_out_of_range_writes_nothing(bad, schedule):
    w = workloads.make_append(seed=5, n_new=[2, 3], seq_lens=[2, 3], Hq=4, Hkv=2, page_size=4,
                              max_pages=2, cos_sin_rows=11, positions=[0, 1, 2, bad, 4])
    r = AppendRun(w, schedule=schedule)
    r.launch()
    assert r.check() == {"flagged": True}


def _wide_block_decode(policy, style, B=128, seed=21):
    """A decode batch of 1,664 latency-schedule warp tasks (128 rows of 12
    quads, plus 128 request tasks): 208 blocks of 8 warps would leave some SMs
    with two blocks, 139 blocks of 12 fit one per SM, so the latency schedule
    takes its wide (12-warp) block here."""
    rng = np.random.default_rng(seed + policy + 3 * style)
    L = rng.integers(1, 400, B)
    return workloads.make_append(seed=seed + policy + 3 * style, n_new=[1] * B, seq_lens=L,
                                 Hq=32, Hkv=8, page_size=16, max_pages=32,
                                 quant_policy=policy, rope_style=style, cos_sin_rows=400,
                                 q_scale_inv=20.0, k_scale=0.05, v_scale=0.05,
                                 qkv_sigma=2.0 if policy else 1.0)


def test_wide_block_preconditions_hold_on_this_device():
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    tasks = 128 * 12 + 128
    assert -(-tasks // 8) > sms and -(-tasks // 12) <= sms, sms
    plan = AppendRun(_wide_block_decode(0, 0), schedule=0).plan()
    assert plan["schedule"] == 1 and plan["block_threads"] == 384 and plan["warp_check"] == 1


# The launch plans of the named workloads on a 148-SM B200: which schedule and
# which latency-schedule variants the parity tests above exercise.
PLANS = {
    "qwen3_decode_bf16": dict(schedule=1, block_threads=384, grid=139, tasks=1664, warp_check=1,
                              bulk_tails=0, request_tails=0),
    "tiny_decode_bf16": dict(schedule=1, block_threads=256, grid=2, tasks=16, warp_check=1,
                             bulk_tails=0, request_tails=1),
    "fp8_decode_dynamic": dict(schedule=1, block_threads=256, tasks=5376, warp_check=0,
                               bulk_tails=1, request_tails=0),
    "decode_out_kv_bf16": dict(schedule=1, block_threads=384, warp_check=1),
    "ragged_prefill_fp8": dict(schedule=2, block_threads=256, grid=296, warp_check=0),
}


@pytest.mark.parametrize("name", sorted(PLANS))
def test_launch_plan_of_named_workloads(name):
    if torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("plans recorded for a 148-SM B200")
    plan = AppendRun(workloads.APPEND_CONFIGS[name](), schedule=0).plan()
    for k, v in PLANS[name].items():
        assert plan[k] == v, (k, plan)


@pytest.mark.parametrize("style", [0, 1])
@pytest.mark.parametrize("policy", [0, 1, 2])
def test_wide_block_decode_parity(policy, style):
    run_and_check(_wide_block_decode(policy, style), schedule=1)


@pytest.mark.parametrize("case", ["non_monotone", "page_table_overrun"])
def test_wide_block_malformed_writes_nothing(case):
    w = _wide_block_decode(1, 0)
    ind, L = w.q_indptr.copy(), w.seq_lens.copy()
    if case == "non_monotone":
        ind[60] = ind[62]
    else:
        L[77] = w.page_size * w.max_pages + 1
    r = AppendRun(w, schedule=1, q_indptr=ind, seq_lens=L)
    r.launch()
    assert r.check() == {"flagged": True}
    assert (r.flags.cpu().numpy() == -1).all()


@pytest.mark.parametrize("policy", [0, 1, 2])
def test_small_tails_owned_by_request_tasks(policy):
    """Tails of at most 4 KiB per request (Hkv 1, page 16) in a one-pass
    latency launch: request tasks zero whole tails, including those of
    requests without new rows and of requests with several rows."""
    n = [1, 3, 0, 1, 0, 17, 1, 2]
    L = [9, 3, 21, 16, 0, 40, 1, 18]
    w = workloads.make_append(seed=30 + policy, n_new=n, seq_lens=L, Hq=8, Hkv=1,
                              page_size=16, max_pages=3, quant_policy=policy, cos_sin_rows=48,
                              q_scale_inv=20.0, k_scale=0.05, v_scale=0.05)
    r, _ = run_and_check(w, schedule=1)
    assert (r.flags.cpu().numpy() == 0).all()


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_largest_batch(schedule):
    B = 16384
    rng = np.random.default_rng(8)
    L = rng.integers(1, 64, B)
    w = workloads.make_append(seed=8, n_new=[1] * B, seq_lens=L, Hq=2, Hkv=1, page_size=16,
                              max_pages=4, quant_policy=1, cos_sin_rows=64, k_scale=0.05,
                              v_scale=0.05)
    run_and_check(w, schedule=schedule)


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_padded_page_stride(schedule):
    w = workloads.make_append(seed=9, n_new=[5, 17, 0, 1], seq_lens=[9, 30, 7, 1], Hq=8,
                              Hkv=2, page_size=16, max_pages=3, quant_policy=2,
                              q_scale_inv=20.0, k_scale=0.05, v_scale=0.05)
    run_and_check(w, page_stride_pad=256, schedule=schedule)


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_every_bf16_input_through_the_fp8_encoder(schedule):
    """All 65536 BF16 codes (inf and NaN included) as Q inputs with no norm and
    an identity rotation (GPT-J, rot_dim 2, position 0), static scale 1: the
    payload is the E4M3 encoding of the input itself, and the GPU's packed
    conversion must equal the oracle's encoder on every code."""
    Hq, Hkv = 8, 1
    per_head = D - 2
    heads = -(-65536 // per_head)
    T = -(-heads // Hq)
    w = workloads.make_append(seed=10, n_new=[1] * T, seq_lens=[1] * T, Hq=Hq, Hkv=Hkv,
                              page_size=4, max_pages=1, quant_policy=2, norm=False, rot_dim=2,
                              rope_style=1, q_scale_inv=1.0, k_scale=1.0, v_scale=1.0)
    codes = np.zeros(T * Hq * per_head, np.uint16)
    codes[:65536] = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    q = w.qkv[:, : Hq * D].reshape(T, Hq, D)
    q[:, :, 2:] = codes.reshape(T, Hq, per_head)
    q[:, :, :2] = 0x3F80                      # the rotated pair stays finite
    w.qkv[:, : Hq * D] = q.reshape(T, Hq * D)
    r, rep = run_and_check(w, schedule=schedule)
    assert rep["q_exact_frac"] == 1.0
    # the payload is the encoding of the input value itself (NaN codes equal)
    got = _np(r.out_q).reshape(T, Hq, D)[:, :, 2:].reshape(-1)[:65536]
    want = oracle.e4m3(bf16_bits_to_f32(codes[:65536]))
    assert (ulp_e4m3(got, want) == 0).all()


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_heads_far_apart_in_scale_normalise_independently(schedule):
    w = workloads.make_append(seed=12, n_new=[3, 2], seq_lens=[40, 2], Hq=16, Hkv=4,
                              page_size=16, max_pages=3, quant_policy=0)
    x = bf16_bits_to_f32(w.qkv).copy()
    for h in range(0, 24, 2):
        x[:, h * D:(h + 1) * D] *= 1e3
    w.qkv = (x.view(np.uint32) >> 16).astype(np.uint16)
    run_and_check(w, schedule=schedule)


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_non_default_stream(schedule):
    w = workloads.tiny_decode_bf16()
    r = AppendRun(w, schedule=schedule)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        r.launch(stream=s)
    s.synchronize()
    r.check()


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_cuda_graph_capture_and_replay_is_bitwise_eager(schedule):
    w = workloads.fp8_decode_dynamic()
    r = AppendRun(w, schedule=schedule)
    r.launch()
    torch.cuda.synchronize()
    eager = (r.out_q.clone(), r.q_scale.clone(), r.k_store.clone(), r.v_store.clone(),
             r.flags.clone())
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        r.launch(stream=s)
    for _ in range(3):
        r.out_q.fill_(0x55)
        r.q_scale.fill_(-1.0)
        r.flags.fill_(7)
        g.replay()
        torch.cuda.synchronize()
        now = (r.out_q, r.q_scale, r.k_store, r.v_store, r.flags)
        for a, b in zip(eager, now):
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    del g
    r.check()


def _special_heads(w, seed):
    """Plant special values into the Q and K heads of w's rows (in place):
    every case lands in a Q head and in a K head of some row."""
    rng = np.random.default_rng(seed)
    D = 128

    def put(r, h, fn):
        head = w.qkv[r, h * D:(h + 1) * D]
        fn(head, rng)

    cases = [
        lambda x, g: x.__setitem__(5, 0x7FC0),                     # NaN, odd slot
        lambda x, g: x.__setitem__(6, 0xFFC1),                     # NaN, even slot
        lambda x, g: x.__setitem__(3, 0x7F80),                     # +Inf
        lambda x, g: x.__setitem__(100, 0xFF80),                   # -Inf
        lambda x, g: x.__setitem__(slice(None), g.choice([0x7F7F, 0xFF7F, 0x7F70], D)),  # ~BF16 max
        lambda x, g: x.__setitem__(slice(None), g.integers(1, 0x80, D)),                  # subnormals
        lambda x, g: x.__setitem__(slice(None), 0),                                      # zeros
        lambda x, g: (x.__setitem__(slice(None), 0), x.__setitem__(77, 0x3F80)),          # one-hot
        lambda x, g: x.__setitem__(slice(None), np.where(g.random(D) < 0.5, 0x7149, 0x0DA2)),  # 1e30 / 1e-30
        lambda x, g: x.__setitem__(slice(None), x & 0x80FF | 0x0080),  # tiny normals
        # the bounds of the fp32-squares form's range: squares near 2^-60
        lambda x, g: x.__setitem__(slice(None), x & 0x807F | 0x3080),
        # values whose fp32 squares round (below 2^-63) beside N(0, 1) values
        lambda x, g: x.__setitem__(slice(None), np.where(g.random(D) < 0.5, x, 0x1CC1)),
        # one square just below the fp32 overflow, then one far above it
        lambda x, g: x.__setitem__(40, 0x5F35),
        lambda x, g: (x.__setitem__(40, 0x5F35), x.__setitem__(41, 0x6780)),
    ]
    heads = list(range(w.Hq)) + list(range(w.Hq, w.Hq + w.Hkv))
    r = 0
    for i, fn in enumerate(cases):
        for h in (heads[i % w.Hq], w.Hq + i % w.Hkv):
            put(r % w.T, h, fn)
            r += 1


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("policy", [0, 1])
def test_special_values_in_normed_heads(policy, schedule):
    """Q/K heads holding NaN (at either conversion slot of a pair), +-Inf,
    values near the BF16 maximum (the mean square overflows), subnormals,
    zeros, a one-hot head, 1e30 beside 1e-30, and tiny normals, against the
    oracle: a NaN makes the whole head NaN, an overflowing mean square gives
    1/sqrt = 0, and everything else matches within the bar."""
    n = [5, 3, 6, 4]
    L = [9, 20, 31, 70]
    w = workloads.make_append(seed=77, n_new=n, seq_lens=L, Hq=16, Hkv=4, page_size=16,
                              max_pages=6, quant_policy=policy, qkv_sigma=1.0,
                              cos_sin_rows=128, k_scale=0.05, v_scale=0.05)
    _special_heads(w, 5)
    _, rep = run_and_check(w, schedule=schedule)
    assert not rep.get("flagged")


@pytest.mark.parametrize("policy", [0, 1])
def test_special_values_in_wide_block_heads(policy):
    """The same special values in a decode batch that takes the latency
    schedule's wide block, whose warps (one task each) form the mean square
    from fp32 squares: its rare-branch fallback against the oracle."""
    w = _wide_block_decode(policy, 0)
    _special_heads(w, 6)
    plan = AppendRun(w, schedule=0).plan()
    assert plan["block_threads"] == 384 and plan["warp_check"] == 1
    _, rep = run_and_check(w, schedule=1)
    assert not rep.get("flagged")
