"""The seeded workloads: determinism, shapes, structure and byte counts."""
import numpy as np
import pytest

import workloads


@pytest.mark.parametrize("name", sorted(workloads.APPEND_CONFIGS))
def test_append_workloads_are_deterministic(name):
    a, b = workloads.APPEND_CONFIGS[name](), workloads.APPEND_CONFIGS[name]()
    for f in ("qkv", "q_indptr", "seq_lens", "page_table", "cos_sin"):
        assert np.array_equal(getattr(a, f), getattr(b, f))


def test_config_shapes():
    c1 = workloads.tiny_decode_bf16()
    assert (c1.T, c1.B, c1.Hq, c1.Hkv, c1.page_size) == (4, 4, 8, 1, 16)
    assert c1.qkv.shape == (4, 1280) and c1.cos_sin.shape == (4096, 128)
    assert sorted(c1.page_table.ravel()) == list(range(64))
    c2 = workloads.qwen3_decode_bf16()
    assert c2.qkv.shape == (128, 6144) and c2.num_pages == 65536
    assert c2.page_table.shape == (128, 512) and c2.cos_sin.shape == (32768, 128)
    assert len(np.unique(c2.page_table)) == 65536
    c3 = workloads.fp8_decode_dynamic()
    assert c3.qkv.shape == (256, 10240) and c3.page_size == 64 and c3.quant_policy == 1
    c4 = workloads.ragged_prefill_fp8()
    n = np.diff(c4.q_indptr)
    assert c4.B == 16 and (n == 0).sum() >= 2 and n.max() <= 2048
    assert np.all(c4.seq_lens >= n) and c4.quant_policy == 2
    assert c4.seq_lens.max() <= c4.max_pages * c4.page_size
    c5 = workloads.mla_decode()
    assert c5.q.shape == (32, 128, 192) and c5.kv_c.shape == (32, 512)
    assert c5.width == 576 and c5.num_blocks == 16384 and c5.rope_style == 1


def test_malformed_indptr_is_non_monotone():
    w = workloads.ragged_prefill_fp8()
    bad = workloads.malformed_indptr(w)
    assert np.any(np.diff(bad) < 0) and bad[0] == 0 and bad[-1] == w.T


def test_byte_counts_match_expected_sizes():
    """Algorithmic bytes per call of the named workloads (order of magnitude
    fixed by the shapes: c2 ~7 MB, c3 ~25 MB with tails the majority)."""
    b2 = workloads.append_bytes(workloads.qwen3_decode_bf16())
    b3 = workloads.append_bytes(workloads.fp8_decode_dynamic())
    assert 6.0e6 < b2["total"] < 8.5e6
    assert 20e6 < b3["total"] < 30e6 and b3["tail_write"] > b3["total"] / 2
    b1 = workloads.append_bytes(workloads.tiny_decode_bf16())
    assert b1["total"] < 60e3


def test_bf16_inputs_are_truncated_normals():
    rng = workloads.rng_for(1)
    bits = workloads.bf16_normal(rng, (1 << 16,), sigma=2.0)
    x = (bits.astype(np.uint32) << 16).view(np.float32)
    assert abs(x.std() - 2.0) < 0.05 and abs(x.mean()) < 0.05
