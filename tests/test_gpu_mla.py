"""GPU parity of fqr_concat_mla_cache against the oracle, through the C ABI:
the full-size MLA decode workload, BF16 and NeoX variants, ragged prefill
with empty requests, malformed metadata, and Q quantised to FP8 (static,
per token, per head, per group of a head's values; bitwise codes and
scales)."""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from tests.gpu_harness import MlaRun


def run(w, **kw):
    r = MlaRun(w, **kw)
    r.launch()
    return r, r.check()


def test_mla_decode_workload_parity():
    r, rep = run(workloads.mla_decode())
    # no norm on this path: both sides evaluate the same fp32 expressions
    assert rep["q_exact_frac"] == 1.0


@pytest.mark.parametrize("fp8", [1, 0])
@pytest.mark.parametrize("style", [1, 0])
def test_mla_small_variants(fp8, style):
    rng = np.random.default_rng(fp8 * 2 + style)
    B = 9
    n = rng.integers(0, 20, B)
    n[3] = 0
    L = rng.integers(0, 100, B) + n
    w = workloads.make_mla(seed=5 + style, n_new=n, seq_lens=L, Hq=13, block_size=16,
                           max_blocks=int(np.ceil(L.max() / 16)) + 1, rope_style=style,
                           cache_fp8=fp8, kv_lora_rank=512, cos_sin_rows=int(L.max()) + 1)
    r, rep = run(w)
    assert rep["q_exact_frac"] == 1.0


@pytest.mark.parametrize("bad", ["non_monotone", "seq_short", "block_overrun", "rows"])
def test_mla_malformed_writes_nothing(bad):
    w = workloads.make_mla(seed=4, n_new=[2, 1, 1], seq_lens=[4, 3, 2], Hq=8, block_size=4,
                           max_blocks=2, kv_lora_rank=64, cos_sin_rows=8)
    over = {"non_monotone": dict(q_indptr=[0, 3, 2, 4]),
            "seq_short": dict(seq_lens=[1, 3, 2]),
            "block_overrun": dict(seq_lens=[9, 3, 2]),
            "rows": dict(seq_lens=[4, 3, 9])}[bad]
    r, rep = run(w, **{k: np.array(v, np.int32) for k, v in over.items()})
    assert rep == {"flagged": True}
    assert (r.flags.cpu().numpy() == -1).all()


def test_mla_graph_replay_matches_eager():
    w = workloads.mla_decode()
    r = MlaRun(w)
    q0 = r.q.clone()
    r.launch()
    torch.cuda.synchronize()
    eager_q, eager_lat = r.q.clone(), r.latent.clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        r.launch(stream=s)
    for _ in range(3):
        r.q.copy_(q0)            # q is rotated in place: restore the input each time
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(r.q, eager_q) and torch.equal(r.latent, eager_lat)
    del g


@pytest.mark.parametrize("q_quant", [1, 2, 3])
def test_mla_decode_q_fp8_parity(q_quant):
    run(workloads.mla_decode(q_quant=q_quant))


@pytest.mark.parametrize("group", [64, 128])
def test_mla_decode_q_fp8_group_parity(group):
    """The full-size MLA decode with per-group Q scales: 3 groups of 64 per
    192-wide head, or 2 (the 128 nope values and the 64 rope values)."""
    run(workloads.mla_decode(q_quant=4, q_group=group))


@pytest.mark.parametrize("group", [8, 16, 24, 64, 96, 128, 192, 256])
@pytest.mark.parametrize("style", [1, 0])
def test_mla_q_fp8_group_ragged(group, style):
    """Ragged batches, empty requests, an all-zero token and an all-zero group
    (floor scales), nope 64 or 128, every group size class: groups inside a
    lane's run, across the nope / rope boundary, longer than the head."""
    rng = np.random.default_rng(group * 2 + style)
    B = 6
    n = rng.integers(0, 25, B)
    n[1] = 0
    L = rng.integers(0, 90, B) + n
    nope = 64 if group % 16 else 128
    w = workloads.make_mla(seed=80 + group + style, n_new=n, seq_lens=L, Hq=19, block_size=16,
                           max_blocks=int(np.ceil(L.max() / 16)) + 1, rope_style=style,
                           nope_dim=nope, kv_lora_rank=128, cos_sin_rows=int(L.max()) + 1,
                           q_quant=4, q_group=group, upper_max=240.0 if style else 448.0)
    w.q[0] = 0                                  # an all-zero token
    w.q[1, 3, :16] = 0                          # a zero run at the start of a head
    run(w)


@pytest.mark.parametrize("q_quant", [1, 2, 3])
@pytest.mark.parametrize("style", [1, 0])
@pytest.mark.parametrize("upper", [448.0, 240.0])
def test_mla_q_fp8_ragged(q_quant, style, upper):
    rng = np.random.default_rng(q_quant * 4 + style)
    B = 7
    n = rng.integers(0, 30, B)
    n[2] = 0
    L = rng.integers(0, 100, B) + n
    w = workloads.make_mla(seed=9 + q_quant, n_new=n, seq_lens=L, Hq=37, block_size=16,
                           max_blocks=int(np.ceil(L.max() / 16)) + 1, rope_style=style,
                           nope_dim=64, kv_lora_rank=256, cos_sin_rows=int(L.max()) + 1,
                           q_quant=q_quant, q_scale_inv=25.0, upper_max=upper)
    w.q[0] = 0                                  # an all-zero token (floor scale)
    run(w)


@pytest.mark.parametrize("style", [1, 0])
def test_mla_q_fp8_per_token_wide_rows_many_clusters(style):
    """Per-token scales with 288 heads (72 quads: the cluster's 64 warps take
    a second quad each for 8 of them) and 50 rows of 1-2 tokens per request
    (more rows than the device holds clusters of one row each)."""
    rng = np.random.default_rng(40 + style)
    B = 30
    n = rng.integers(1, 3, B)
    L = rng.integers(2, 300, B) + n
    w = workloads.make_mla(seed=41 + style, n_new=n, seq_lens=L, Hq=288, block_size=64,
                           max_blocks=int(np.ceil(L.max() / 64)) + 1, rope_style=style,
                           kv_lora_rank=512, cos_sin_rows=int(L.max()) + 1, q_quant=2,
                           upper_max=448.0)
    assert w.T >= 40
    w.q[3] = 0                                  # an all-zero token (floor scale)
    run(w)


@pytest.mark.parametrize("q_quant", [1, 2, 3, 4])
def test_mla_q_fp8_with_bf16_latent(q_quant):
    """FP8 Q with a BF16 latent cache (every kernel variant's FP8 = 0 side)."""
    rng = np.random.default_rng(60 + q_quant)
    n = rng.integers(1, 4, 6)
    L = rng.integers(1, 90, 6) + n
    w = workloads.make_mla(seed=61 + q_quant, n_new=n, seq_lens=L, Hq=20, block_size=32,
                           max_blocks=int(np.ceil(L.max() / 32)) + 1, kv_lora_rank=128,
                           cos_sin_rows=int(L.max()) + 1, cache_fp8=0, q_quant=q_quant,
                           q_scale_inv=25.0, q_group=64)
    run(w)


@pytest.mark.parametrize("Hq", [4, 8, 20])
def test_mla_q_fp8_per_token_few_heads(Hq):
    """Per-token scales with fewer quads than the cluster has blocks: the
    blocks without a quad still take part in the cluster's maximum."""
    rng = np.random.default_rng(70 + Hq)
    n = rng.integers(1, 3, 5)
    L = rng.integers(1, 60, 5) + n
    w = workloads.make_mla(seed=71 + Hq, n_new=n, seq_lens=L, Hq=Hq, block_size=16,
                           max_blocks=int(np.ceil(L.max() / 16)) + 1, kv_lora_rank=64,
                           cos_sin_rows=int(L.max()) + 1, q_quant=2)
    run(w)


@pytest.mark.parametrize("q_quant", [1, 2, 3, 4])
def test_mla_q_fp8_malformed_writes_nothing(q_quant):
    w = workloads.make_mla(seed=4, n_new=[2, 1, 1], seq_lens=[4, 3, 2], Hq=8, block_size=4,
                           max_blocks=2, kv_lora_rank=64, cos_sin_rows=8, q_quant=q_quant,
                           q_group=32)
    r, rep = run(w, q_indptr=np.array([0, 3, 2, 4], np.int32))
    assert rep == {"flagged": True}
    assert torch.equal(r.q_out, r.q_out_before)


@pytest.mark.parametrize("graph", [False, True])
def test_back_to_back_launches_read_each_others_writes(graph):
    """Two fqr_concat_mla_cache launches on one stream with nothing in between
    (each launch lets the next start its prologue early: programmatic
    dependent launch, also inside a CUDA graph).  The second reads the q the
    first rotated in place, so q ends up rotated twice: exactly the oracle
    applied twice.  A launch that read q before the preceding launch had
    finished would leave it rotated once."""
    import oracle
    from tests.gpu_harness import _np
    rng = np.random.default_rng(90)
    n = rng.integers(1, 4, 24)
    L = rng.integers(1, 3000, 24) + n
    w = workloads.make_mla(seed=91, n_new=n, seq_lens=L, Hq=128, block_size=64,
                           max_blocks=int(np.ceil(L.max() / 64)) + 1, kv_lora_rank=512,
                           cos_sin_rows=int(L.max()) + 1)
    r = MlaRun(w)
    lat0 = _np(r.latent).copy()
    if graph:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            r.launch(stream=s)
            r.launch(stream=s)
        g.replay()
    else:
        r.launch()
        r.launch()
    torch.cuda.synchronize()
    q, lat, fl = w.q.copy(), lat0.copy(), np.zeros(w.B, np.int32)
    for _ in range(2):
        assert oracle.concat_mla_cache(w, q, lat, fl) == 0
    assert np.array_equal(_np(r.q), q)
    assert np.array_equal(_np(r.latent), lat)
    assert not r.flags.cpu().numpy().any()
    assert not np.array_equal(q, w.q)
    if graph:
        del g
