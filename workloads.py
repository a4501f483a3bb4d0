"""Seeded synthetic inputs for the fused QK-norm + RoPE + quant + paged-append
path and for the MLA latent concat.

This module only draws inputs.  It holds none of the method's arithmetic:
BF16 inputs are made by truncating float32 normal draws to their top 16 bits,
and the cos/sin cache (an input of the method, looked up by position) is
tabulated in float64 and rounded once to float32 by numpy.  Both the oracle
side and the CUDA side of every test and of bench.py take their inputs from
here, as host numpy arrays.

The five named workloads follow the shapes, distributions and structure of the
pages' workloads (FlashInfer PR #5956 "Performance" rows: decode with one token
per request, ragged prefill with empty requests and cross-page appends, random
page tables; the vLLM issue #24678 model table for the DeepSeek-R1 MLA shape).
"""
from __future__ import annotations

import functools
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

HEAD_DIM = 128


def rng_for(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def bf16_normal(rng: np.random.Generator, shape, mean=0.0, sigma=1.0) -> np.ndarray:
    """BF16 bit patterns (uint16) of float32 N(mean, sigma) draws, truncated."""
    x = (rng.standard_normal(size=shape, dtype=np.float32) * np.float32(sigma)
         + np.float32(mean)).astype(np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def cos_sin_cache(rows: int, rot: int, theta: float) -> np.ndarray:
    """fp32 [rows, rot] = [cos(p * f_i) | sin(p * f_i)], f_i = theta^(-2i/rot).

    Tabulated in float64 and rounded once to float32; row 0 is exactly
    [1, ..., 1 | 0, ..., 0].  Returns a fresh copy (tables are memoised)."""
    return _cos_sin_cache(int(rows), int(rot), float(theta)).copy()


@functools.lru_cache(maxsize=16)
def _cos_sin_cache(rows: int, rot: int, theta: float) -> np.ndarray:
    half = rot // 2
    inv_freq = theta ** (-(np.arange(half, dtype=np.float64) * 2.0) / rot)
    ang = np.arange(rows, dtype=np.float64)[:, None] * inv_freq[None, :]
    return np.concatenate([np.cos(ang), np.sin(ang)], axis=1).astype(np.float32)


@dataclass
class AppendWorkload:
    name: str
    seed: int
    T: int
    B: int
    Hq: int
    Hkv: int
    qkv: np.ndarray            # uint16 [T, row_stride]
    row_stride: int
    q_norm_w: Optional[np.ndarray]   # uint16 [128] or None
    k_norm_w: Optional[np.ndarray]
    eps: float
    cos_sin: np.ndarray        # float32 [rows, rot_dim]
    rot_dim: int
    rope_style: int            # 0 NeoX, 1 GPT-J
    positions: Optional[np.ndarray]  # int64 [T] or None
    q_indptr: np.ndarray       # int32 [B + 1]
    seq_lens: np.ndarray       # int32 [B]
    page_table: np.ndarray     # int32 [B, max_pages]
    num_pages: int
    page_size: int
    quant_policy: int
    q_scale_inv: float = 1.0
    k_scale: float = 1.0
    v_scale: float = 1.0
    upper_max: float = 448.0
    max_seqlen: int = 0        # policy 1: > 0 selects the prefill q_scale layout
    norm_style: int = 0        # 0: x_hat * w, 1 (Gemma): x_hat * (1 + w)
    out_kv: bool = False       # K/V to caller-owned [T, Hkv, 128] buffers
    gate_heads: int = 0        # G heads after V in each row (never read)
    extra: dict = field(default_factory=dict)

    @property
    def cos_sin_rows(self) -> int:
        return int(self.cos_sin.shape[0])

    @property
    def max_pages(self) -> int:
        return int(self.page_table.shape[1])

    @property
    def kv_esize(self) -> int:
        return 2 if self.quant_policy == 0 else 1

    @property
    def q_scale_shape(self) -> tuple:
        """Decode layout [T, Hq]; with max_seqlen > 0 the prefill layout
        [B, Hq, round_up(max_seqlen, 128)]."""
        if self.max_seqlen > 0:
            return (self.B, self.Hq, -(-self.max_seqlen // 128) * 128)
        return (self.T, self.Hq)

    @property
    def q_esize(self) -> int:
        return 2 if self.quant_policy == 0 else 1


@dataclass
class MlaWorkload:
    name: str
    seed: int
    T: int
    B: int
    Hq: int
    nope_dim: int
    rope_dim: int
    q: np.ndarray              # uint16 [T, Hq, nope + rope]
    kv_c: np.ndarray           # uint16 [T, kv_lora_rank]
    k_pe: np.ndarray           # uint16 [T, rope_dim]
    cos_sin: np.ndarray        # float32 [rows, rope_dim]
    rope_style: int
    positions: Optional[np.ndarray]
    q_indptr: np.ndarray
    seq_lens: np.ndarray
    block_table: np.ndarray    # int32 [B, max_blocks]
    num_blocks: int
    block_size: int
    cache_fp8: int
    kv_scale: float
    q_quant: int = 0           # 0 none, 1 static, 2 dynamic per token, 3 per head, 4 per group
    q_scale_inv: float = 1.0
    upper_max: float = 448.0
    q_group: int = 0           # q_quant 4: values per group of a head

    @property
    def q_scale_shape(self) -> tuple:
        """[T] per token, [T, Hq] per head, [T, Hq, ceil(W / q_group)] per group."""
        W = self.nope_dim + self.rope_dim
        return {2: (self.T,), 3: (self.T, self.Hq),
                4: (self.T, self.Hq, -(-W // max(1, self.q_group)))}.get(self.q_quant, (1,))

    @property
    def kv_lora_rank(self) -> int:
        return int(self.kv_c.shape[1])

    @property
    def cos_sin_rows(self) -> int:
        return int(self.cos_sin.shape[0])

    @property
    def max_blocks(self) -> int:
        return int(self.block_table.shape[1])

    @property
    def width(self) -> int:
        return self.kv_lora_rank + self.rope_dim


def make_append(*, name="custom", seed=0, n_new, seq_lens, Hq, Hkv, page_size,
                max_pages, num_pages=None, quant_policy=0, qkv_sigma=1.0,
                norm=True, rot_dim=HEAD_DIM, rope_style=0, theta=1e6,
                cos_sin_rows=None, row_pad=0, positions=None,
                q_scale_inv=1.0, k_scale=1.0, v_scale=1.0, upper_max=448.0,
                eps=1e-6, max_seqlen=0, norm_style=0, out_kv=False,
                gate_heads=0) -> AppendWorkload:
    """Build a paged-append workload from per-request new-token counts and
    post-append lengths.  The page table is a seeded random permutation of
    `num_pages` page ids reshaped to [B, max_pages] (num_pages defaults to
    B * max_pages).  `gate_heads` appends that many 128-wide G heads to every
    row ([Q | K | V | G]), ahead of any `row_pad`."""
    rng = rng_for(seed)
    n_new = np.asarray(n_new, dtype=np.int64)
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    B = int(len(n_new))
    T = int(n_new.sum())
    q_indptr = np.zeros(B + 1, dtype=np.int32)
    q_indptr[1:] = np.cumsum(n_new)
    H = Hq + 2 * Hkv
    row_stride = (H + gate_heads) * HEAD_DIM + row_pad
    qkv = bf16_normal(rng, (T, row_stride), sigma=qkv_sigma)
    qw = bf16_normal(rng, (HEAD_DIM,), mean=1.0, sigma=0.1) if norm else None
    kw = bf16_normal(rng, (HEAD_DIM,), mean=1.0, sigma=0.1) if norm else None
    if num_pages is None:
        num_pages = B * max_pages
    perm = rng.permutation(num_pages).astype(np.int32)
    if num_pages >= B * max_pages:
        page_table = perm[: B * max_pages].reshape(B, max_pages).copy()
    else:  # fewer pages than table slots: pad with ids from the permutation
        page_table = np.resize(perm, B * max_pages).reshape(B, max_pages).copy()
    if cos_sin_rows is None:
        cos_sin_rows = max(int(seq_lens.max(initial=1)), 1)
    cs = cos_sin_cache(cos_sin_rows, rot_dim, theta)
    if positions is not None:
        positions = np.asarray(positions, dtype=np.int64)
    return AppendWorkload(
        name=name, seed=seed, T=T, B=B, Hq=Hq, Hkv=Hkv, qkv=qkv,
        row_stride=row_stride, q_norm_w=qw, k_norm_w=kw, eps=eps, cos_sin=cs,
        rot_dim=rot_dim, rope_style=rope_style, positions=positions,
        q_indptr=q_indptr, seq_lens=seq_lens, page_table=page_table,
        num_pages=num_pages, page_size=page_size, quant_policy=quant_policy,
        q_scale_inv=q_scale_inv, k_scale=k_scale, v_scale=v_scale,
        upper_max=upper_max, max_seqlen=max_seqlen, norm_style=norm_style,
        out_kv=out_kv, gate_heads=gate_heads)


def tiny_decode_bf16(seed=1001) -> AppendWorkload:
    """4 requests, one new token each, Hq 8 / Hkv 1, page 16, BF16 cache."""
    rng = rng_for(seed + 7)
    L = rng.integers(1, 256, size=4, endpoint=True)
    return make_append(name="tiny_decode_bf16_B4_h8x1_p16", seed=seed,
                       n_new=[1] * 4, seq_lens=L, Hq=8, Hkv=1, page_size=16,
                       max_pages=16, quant_policy=0, cos_sin_rows=4096)


def qwen3_decode_bf16(seed=1002) -> AppendWorkload:
    """Qwen3-style decode: 128 requests x 1 token, Hq 32 / Hkv 8, page 16,
    1M-slot BF16 NHD cache [65536, 16, 8, 128], 32768 cos/sin rows."""
    rng = rng_for(seed + 7)
    L = rng.integers(1, 8192, size=128, endpoint=True)
    return make_append(name="qwen3_decode_bf16_B128_h32x8_p16", seed=seed,
                       n_new=[1] * 128, seq_lens=L, Hq=32, Hkv=8, page_size=16,
                       max_pages=512, num_pages=65536, quant_policy=0,
                       cos_sin_rows=32768)


def fp8_decode_dynamic(seed=1003) -> AppendWorkload:
    """FP8 decode with a dynamic per-token/per-head Q scale: 256 x 1 token,
    Hq 64 / Hkv 8, qkv N(0, sigma=2), page 64, FP8 cache [65536, 64, 8, 128]."""
    rng = rng_for(seed + 7)
    L = rng.integers(1, 16384, size=256, endpoint=True)
    return make_append(name="fp8_decode_dynq_B256_h64x8_p64", seed=seed,
                       n_new=[1] * 256, seq_lens=L, Hq=64, Hkv=8, page_size=64,
                       max_pages=256, num_pages=65536, quant_policy=1,
                       qkv_sigma=2.0, cos_sin_rows=16384, k_scale=0.05,
                       v_scale=0.05, upper_max=448.0)


def ragged_prefill_fp8(seed=1004, n_new=None) -> AppendWorkload:
    """Ragged prefill, static FP8: 16 requests with U[0, 2048] new tokens (two
    forced empty) on U[0, 4096] prior context, page 16, Hq 64 / Hkv 8.
    n_new: keep these per-request token counts instead of the drawn ones (a
    batch of the same shape with other data, positions and pages)."""
    rng = rng_for(seed + 7)
    n = rng.integers(0, 2048, size=16, endpoint=True)
    n[rng.choice(16, size=2, replace=False)] = 0
    if n_new is not None:
        n = np.asarray(n_new, dtype=np.int64).copy()
    prior = rng.integers(0, 4096, size=16, endpoint=True)
    L = prior + n
    return make_append(name="ragged_prefill_fp8_B16_h64x8_p16", seed=seed,
                       n_new=n, seq_lens=L, Hq=64, Hkv=8, page_size=16,
                       max_pages=384, quant_policy=2, cos_sin_rows=8192,
                       q_scale_inv=1.0 / 0.05, k_scale=0.05, v_scale=0.05)


def malformed_indptr(w: AppendWorkload, seed=1104) -> np.ndarray:
    """A non-monotone copy of w.q_indptr: one interior entry raised above its
    successor."""
    rng = rng_for(seed)
    ind = w.q_indptr.copy()
    if w.B < 2:
        raise ValueError("needs at least two requests")
    j = int(rng.integers(1, w.B))          # interior entry 1..B-1
    ind[j] = ind[j + 1] + 1 + int(rng.integers(0, 8))
    return ind


def mla_decode(seed=1005, q_quant=0, q_group=0) -> MlaWorkload:
    """MLA decode latent concat: 32 x 1 token, 128 query heads, q [32,128,192]
    with interleaved RoPE on dims 128..191 (theta 10000), kv_c [32, 512],
    k_pe [32, 64], FP8 latent cache [16384, 64, 576] with scale 0.02.
    q_quant > 0: the same call with Q quantised to FP8 E4M3 (1 static
    per-tensor with q_scale_inv 1/0.02, 2 dynamic per token, 3 per head,
    4 per group of q_group values of a head)."""
    rng = rng_for(seed)
    B = T = 32
    Hq, nope, rope_dim, rank = 128, 128, 64, 512
    q = bf16_normal(rng, (T, Hq, nope + rope_dim))
    kv_c = bf16_normal(rng, (T, rank))
    k_pe = bf16_normal(rng, (T, rope_dim))
    L = rng.integers(1, 32768, size=B, endpoint=True).astype(np.int32)
    block_size, max_blocks = 64, 512
    num_blocks = B * max_blocks
    perm = rng.permutation(num_blocks).astype(np.int32).reshape(B, max_blocks)
    cs = cos_sin_cache(32768, rope_dim, 10000.0)
    q_indptr = np.arange(B + 1, dtype=np.int32)
    suffix = {0: "", 1: "_qfp8_static", 2: "_qfp8_token", 3: "_qfp8_head",
              4: f"_qfp8_group{q_group}"}[q_quant]
    return MlaWorkload(name="mla_decode_B32_h128_latent576_fp8" + suffix, seed=seed,
                       T=T, B=B, Hq=Hq, nope_dim=nope, rope_dim=rope_dim, q=q,
                       kv_c=kv_c, k_pe=k_pe, cos_sin=cs, rope_style=1,
                       positions=None, q_indptr=q_indptr, seq_lens=L,
                       block_table=perm.copy(), num_blocks=num_blocks,
                       block_size=block_size, cache_fp8=1, kv_scale=0.02,
                       q_quant=q_quant, q_scale_inv=1 / 0.02, q_group=q_group)


def make_mla(*, seed=0, n_new, seq_lens, Hq, block_size, max_blocks,
             num_blocks=None, nope_dim=128, rope_dim=64, kv_lora_rank=512,
             rope_style=1, theta=10000.0, cos_sin_rows=None, cache_fp8=1,
             kv_scale=0.02, positions=None, q_quant=0, q_scale_inv=1.0,
             upper_max=448.0, q_group=0) -> MlaWorkload:
    rng = rng_for(seed)
    n_new = np.asarray(n_new, dtype=np.int64)
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    B, T = len(n_new), int(n_new.sum())
    q_indptr = np.zeros(B + 1, dtype=np.int32)
    q_indptr[1:] = np.cumsum(n_new)
    q = bf16_normal(rng, (T, Hq, nope_dim + rope_dim))
    kv_c = bf16_normal(rng, (T, kv_lora_rank))
    k_pe = bf16_normal(rng, (T, rope_dim))
    if num_blocks is None:
        num_blocks = B * max_blocks
    perm = rng.permutation(num_blocks).astype(np.int32)
    table = np.resize(perm, B * max_blocks).reshape(B, max_blocks).copy()
    if cos_sin_rows is None:
        cos_sin_rows = max(int(seq_lens.max(initial=1)), 1)
    cs = cos_sin_cache(cos_sin_rows, rope_dim, theta)
    if positions is not None:
        positions = np.asarray(positions, dtype=np.int64)
    return MlaWorkload(name="mla_custom", seed=seed, T=T, B=B, Hq=Hq,
                       nope_dim=nope_dim, rope_dim=rope_dim, q=q, kv_c=kv_c,
                       k_pe=k_pe, cos_sin=cs, rope_style=rope_style,
                       positions=positions, q_indptr=q_indptr,
                       seq_lens=seq_lens, block_table=table,
                       num_blocks=num_blocks, block_size=block_size,
                       cache_fp8=cache_fp8, kv_scale=kv_scale, q_quant=q_quant,
                       q_scale_inv=q_scale_inv, upper_max=upper_max, q_group=q_group)


def prefill_dynq_gemma(seed=1006, q_len=129) -> AppendWorkload:
    """Dynamic-Q prefill with the [B, Hq, round_up(max_seqlen, 128)] q_scale
    layout and the Gemma-style norm: 4 requests x q_len new tokens each,
    max_seqlen = q_len (the pages' padding-edge rows use q_len 127 / 128 /
    129), Hq 64 / Hkv 8, page 64, prior context U[0, 1024], k/v scale 0.05."""
    rng = rng_for(seed + 7)
    prior = rng.integers(0, 1024, size=4, endpoint=True)
    L = prior + q_len
    return make_append(name=f"prefill_dynq_gemma_B4_q{q_len}_h64x8_p64", seed=seed,
                       n_new=[q_len] * 4, seq_lens=L, Hq=64, Hkv=8, page_size=64,
                       max_pages=64, num_pages=4096, quant_policy=1,
                       cos_sin_rows=2048, k_scale=0.05, v_scale=0.05,
                       max_seqlen=q_len, norm_style=1)


def decode_out_kv_bf16(seed=1007) -> AppendWorkload:
    """Decode into caller-owned K/V buffers (no paged cache, no tail): 128
    requests x 1 token, Hq 32 / Hkv 8, BF16."""
    rng = rng_for(seed + 7)
    L = rng.integers(1, 8192, size=128, endpoint=True)
    return make_append(name="decode_out_kv_bf16_B128_h32x8", seed=seed,
                       n_new=[1] * 128, seq_lens=L, Hq=32, Hkv=8, page_size=16,
                       max_pages=512, num_pages=1, quant_policy=0,
                       cos_sin_rows=8192, out_kv=True)


def gate_tail_decode_bf16(seed=1008) -> AppendWorkload:
    """Gated-attention rows [Q | K | V | G] (one G head per Q head, left
    untouched): 128 requests x 1 token, Hq 32 / Hkv 4, page 16, BF16 cache."""
    rng = rng_for(seed + 7)
    L = rng.integers(1, 8192, size=128, endpoint=True)
    return make_append(name="gate_tail_decode_bf16_B128_h32x4g32_p16", seed=seed,
                       n_new=[1] * 128, seq_lens=L, Hq=32, Hkv=4, page_size=16,
                       max_pages=512, num_pages=65536, quant_policy=0,
                       cos_sin_rows=8192, gate_heads=32)


APPEND_CONFIGS = {
    "tiny_decode_bf16": tiny_decode_bf16,
    "qwen3_decode_bf16": qwen3_decode_bf16,
    "fp8_decode_dynamic": fp8_decode_dynamic,
    "ragged_prefill_fp8": ragged_prefill_fp8,
    "prefill_dynq_gemma": prefill_dynq_gemma,
    "decode_out_kv_bf16": decode_out_kv_bf16,
    "gate_tail_decode_bf16": gate_tail_decode_bf16,
}
MLA_CONFIGS = {"mla_decode": mla_decode,
               "mla_decode_qfp8_static": lambda seed=1005: mla_decode(seed, q_quant=1),
               "mla_decode_qfp8_token": lambda seed=1005: mla_decode(seed, q_quant=2),
               "mla_decode_qfp8_head": lambda seed=1005: mla_decode(seed, q_quant=3),
               "mla_decode_qfp8_group64": lambda seed=1005: mla_decode(seed, q_quant=4,
                                                                       q_group=64),
               "mla_decode_qfp8_group128": lambda seed=1005: mla_decode(seed, q_quant=4,
                                                                        q_group=128)}


# ---------------------------------------------------------------------------
# Algorithmic bytes (what the method itself must move; tail zeros count)
# ---------------------------------------------------------------------------

def append_bytes(w: AppendWorkload) -> dict:
    """Bytes a fused append must read and write: packed Q/K/V heads (row
    padding excluded), norm weights, one cos/sin row per token, metadata, the
    pages' table entries, out_q, K/V rows, last-page tail zeros, q_scale and
    flags."""
    D = HEAD_DIM
    T, B, Hq, Hkv = w.T, w.B, w.Hq, w.Hkv
    P = w.page_size
    reads = T * (Hq + 2 * Hkv) * D * 2
    reads += (2 * D * 2) if w.q_norm_w is not None else 0
    reads += T * w.rot_dim * 4
    reads += 4 * (B + 1) + 4 * B
    # one page-table entry per distinct (request, page) touched (none when
    # K/V go to caller-owned buffers)
    touched = 0
    for b in range(B if not w.out_kv else 0):
        lo, hi, L = int(w.q_indptr[b]), int(w.q_indptr[b + 1]), int(w.seq_lens[b])
        pages = set()
        for r in range(lo, hi):
            pages.add((r + L - hi) // P)
        if L > 0:
            pages.add((L - 1) // P)
        touched += len(pages)
    reads += 4 * touched
    if w.positions is not None:
        reads += 8 * T
    bq, bkv = w.q_esize, w.kv_esize
    writes = T * Hq * D * bq + T * 2 * Hkv * D * bkv
    tail_rows = 0
    for b in range(B if not w.out_kv else 0):   # no tail without paged caches
        L = int(w.seq_lens[b])
        if L > 0:
            tail_rows += P - 1 - (L - 1) % P
    writes += tail_rows * 2 * Hkv * D * bkv
    if w.quant_policy == 1:
        writes += T * Hq * 4
    writes += 4 * B
    return {"read": int(reads), "write": int(writes), "total": int(reads + writes),
            "tail_write": int(tail_rows * 2 * Hkv * D * bkv)}


def mla_bytes(w: MlaWorkload) -> dict:
    T, B = w.T, w.B
    W = w.nope_dim + w.rope_dim
    if w.q_quant:   # the whole head read, quantised into q_out (one byte each)
        reads = T * w.Hq * W * 2
        writes = T * w.Hq * W + 4 * int(np.prod(w.q_scale_shape)) * (w.q_quant >= 2)
    else:           # the rope part rotated in place
        reads = T * w.Hq * w.rope_dim * 2
        writes = T * w.Hq * w.rope_dim * 2
    reads += T * (w.kv_lora_rank + w.rope_dim) * 2
    reads += T * w.rope_dim * 4                  # cos/sin row
    reads += 4 * (B + 1) + 4 * B + 4 * T         # metadata + one table entry per token
    cache_e = 1 if w.cache_fp8 else 2
    writes += T * w.width * cache_e + 4 * B
    return {"read": int(reads), "write": int(writes), "total": int(reads + writes)}


def shrink_cache(w: AppendWorkload, max_len: int = 1024) -> AppendWorkload:
    """A copy of a decode-style workload on a smaller cache, for profiling.

    Post-append lengths wrap modulo max_len (a multiple of the page size), so
    every request keeps its position inside its last page -- hence the same
    tail size and the same bytes per call -- while the page table and the
    cache shrink to max_len / page_size pages per request."""
    import copy
    if max_len % w.page_size:
        raise ValueError("max_len must be a multiple of the page size")
    n = np.diff(w.q_indptr)
    L = w.seq_lens.astype(np.int64)
    L2 = np.where(L > 0, (L - 1) % max_len + 1, 0)
    if np.any(L2 < n):
        raise ValueError("a request appends more rows than max_len")
    s = copy.copy(w)
    s.seq_lens = L2.astype(np.int32)
    mp = max_len // w.page_size
    rng = rng_for(w.seed + 99)
    s.num_pages = w.B * mp
    s.page_table = rng.permutation(s.num_pages).astype(np.int32).reshape(w.B, mp)
    s.cos_sin = w.cos_sin[:max_len].copy()
    return s
