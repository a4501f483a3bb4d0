"""Pins of the oracle's MLA latent concat: Q rope part rotated in place (nope
part untouched), latent rows [kv_c | rope(k_pe)] / scale at the slot an
inverse-direction model predicts, nothing else written, and validation."""
import math

import numpy as np
import pytest

import oracle
import workloads
from tests._util import bf16_bits_to_f32, bf16_rne_torch, e4m3_brute


def run(w, fill_seed=2, **over):
    rng = np.random.default_rng(fill_seed)
    dt = np.uint8 if w.cache_fp8 else np.uint16
    lat = rng.integers(0, 256 if w.cache_fp8 else 65536,
                       size=(w.num_blocks, w.block_size, w.width)).astype(dt)
    lat0 = lat.copy()
    q = w.q.copy()
    flags = np.full(w.B, 77, np.int32)
    rc = oracle.concat_mla_cache(w, q, lat, flags, **over)
    return rc, q, lat0, lat, flags


def expected_latent_row(w, r, pos):
    kv = bf16_bits_to_f32(w.kv_c[r])
    kpe = oracle.rope(bf16_bits_to_f32(w.k_pe[r]), w.cos_sin[pos], w.rope_style)
    if w.cache_fp8:
        s = np.float32(w.kv_scale)
        return np.concatenate([e4m3_brute((kv / s).astype(np.float32)),
                               e4m3_brute((kpe / s).astype(np.float32))])
    return np.concatenate([w.kv_c[r], bf16_rne_torch(kpe)])


def check(w, q, lat0, lat):
    n_new = np.diff(w.q_indptr)
    bs = w.block_size
    owner = {}
    for b in range(w.B):
        for k in range(math.ceil(int(w.seq_lens[b]) / bs)):
            owner[int(w.block_table[b, k])] = (b, k)
    # Q
    for b in range(w.B):
        lo, hi, L = int(w.q_indptr[b]), int(w.q_indptr[b + 1]), int(w.seq_lens[b])
        for r in range(lo, hi):
            pos = int(w.positions[r]) if w.positions is not None else r + L - hi
            assert np.array_equal(q[r, :, :w.nope_dim], w.q[r, :, :w.nope_dim])
            for h in range(w.Hq):
                y = oracle.rope(bf16_bits_to_f32(w.q[r, h, w.nope_dim:]), w.cos_sin[pos],
                                w.rope_style)
                assert np.array_equal(q[r, h, w.nope_dim:], bf16_rne_torch(y))
    # latent rows
    for g in range(w.num_blocks):
        for j in range(bs):
            if g in owner:
                b, k = owner[g]
                p, L, n = k * bs + j, int(w.seq_lens[b]), int(n_new[b])
                if L - n <= p < L:
                    r = int(w.q_indptr[b]) + p - (L - n)
                    pos = int(w.positions[r]) if w.positions is not None else p
                    assert np.array_equal(lat[g, j], expected_latent_row(w, r, pos)), (g, j)
                    continue
            assert np.array_equal(lat[g, j], lat0[g, j]), (g, j)


@pytest.mark.parametrize("fp8", [1, 0])
@pytest.mark.parametrize("style", [1, 0])
def test_mla_decode_small(fp8, style):
    w = workloads.make_mla(seed=9, n_new=[1, 1, 1], seq_lens=[5, 1, 17], Hq=4,
                           block_size=4, max_blocks=5, rope_style=style, cache_fp8=fp8,
                           kv_lora_rank=64, cos_sin_rows=20)
    rc, q, lat0, lat, fl = run(w)
    assert rc == 0 and not fl.any()
    check(w, q, lat0, lat)


def test_mla_ragged_prefill_with_empty_requests():
    w = workloads.make_mla(seed=10, n_new=[3, 0, 5, 2], seq_lens=[3, 7, 9, 12], Hq=2,
                           block_size=4, max_blocks=3, kv_lora_rank=32, cos_sin_rows=12)
    rc, q, lat0, lat, fl = run(w)
    assert rc == 0 and not fl.any()
    check(w, q, lat0, lat)


def test_mla_position_zero_leaves_rope_part_unrotated():
    w = workloads.make_mla(seed=3, n_new=[1], seq_lens=[1], Hq=2, block_size=4,
                           max_blocks=1, kv_lora_rank=16)
    rc, q, _, _, _ = run(w)
    assert rc == 0 and np.array_equal(q, w.q)


@pytest.mark.parametrize("bad", ["non_monotone", "seq_short", "block_overrun"])
def test_mla_malformed_flags_and_writes_nothing(bad):
    w = workloads.make_mla(seed=4, n_new=[2, 1, 1], seq_lens=[4, 3, 2], Hq=2,
                           block_size=4, max_blocks=2, kv_lora_rank=16, cos_sin_rows=8)
    over = {"non_monotone": dict(q_indptr=np.array([0, 3, 2, 4], np.int32)),
            "seq_short": dict(seq_lens=np.array([1, 3, 2], np.int32)),
            "block_overrun": dict(seq_lens=np.array([9, 3, 2], np.int32))}[bad]
    rc, q, lat0, lat, fl = run(w, **over)
    assert rc == 1 and list(fl) == [-1] * 3
    assert np.array_equal(q, w.q) and np.array_equal(lat, lat0)
