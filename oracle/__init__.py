"""ctypes front-end of the CPU oracle (oracle/fqr_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
cpu_baseline / reference legs of bench.py.  The product path
(qk_norm_rope_token_b200) never imports it.

All arrays are host numpy arrays.  BF16 values are uint16 bit patterns, FP8
E4M3 values uint8 codes.  Functions that write modify their arguments in place.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

from . import build as _build

_LIB = None

c_i32, c_i64, c_f32, c_vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p


class _AppendArgs(ctypes.Structure):
    _fields_ = [
        ("qkv", c_vp), ("row_stride", c_i64),
        ("T", c_i32), ("B", c_i32), ("Hq", c_i32), ("Hkv", c_i32),
        ("q_norm_w", c_vp), ("k_norm_w", c_vp), ("eps", c_f32),
        ("cos_sin", c_vp), ("cos_sin_rows", c_i32), ("rot_dim", c_i32),
        ("rope_style", c_i32), ("positions", c_vp),
        ("q_indptr", c_vp), ("seq_lens", c_vp), ("page_table", c_vp),
        ("max_pages", c_i32), ("num_pages", c_i32), ("page_size", c_i32),
        ("quant_policy", c_i32),
        ("q_scale_inv", c_f32), ("k_scale", c_f32), ("v_scale", c_f32),
        ("upper_max", c_f32),
        ("k_cache", c_vp), ("v_cache", c_vp),
        ("k_page_stride", c_i64), ("v_page_stride", c_i64),
        ("out_q", c_vp), ("q_scale", c_vp), ("flags", c_vp),
        ("max_seqlen", c_i32), ("norm_style", c_i32), ("out_k", c_vp), ("out_v", c_vp),
    ]


class _MlaArgs(ctypes.Structure):
    _fields_ = [
        ("q", c_vp), ("T", c_i32), ("B", c_i32), ("Hq", c_i32),
        ("nope_dim", c_i32), ("rope_dim", c_i32),
        ("q_token_stride", c_i64), ("q_head_stride", c_i64),
        ("kv_c", c_vp), ("kv_lora_rank", c_i32), ("kv_c_stride", c_i64),
        ("k_pe", c_vp), ("k_pe_stride", c_i64),
        ("cos_sin", c_vp), ("cos_sin_rows", c_i32), ("rope_style", c_i32),
        ("positions", c_vp), ("q_indptr", c_vp), ("seq_lens", c_vp),
        ("block_table", c_vp), ("max_blocks", c_i32),
        ("latent_cache", c_vp), ("num_blocks", c_i32), ("block_size", c_i32),
        ("cache_fp8", c_i32), ("kv_scale", c_f32), ("flags", c_vp),
        ("q_quant", c_i32), ("q_scale_inv", c_f32), ("upper_max", c_f32),
        ("q_out", c_vp), ("q_scale", c_vp), ("q_group", c_i32),
    ]


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.fqro_f32_to_e4m3_rn_satfinite.restype = ctypes.c_uint8
        L.fqro_f32_to_e4m3_rn_satfinite.argtypes = [c_f32]
        L.fqro_f32_to_bf16_rne.restype = ctypes.c_uint16
        L.fqro_f32_to_bf16_rne.argtypes = [c_f32]
        L.fqro_f32_to_e4m3_array.argtypes = [c_vp, c_vp, c_i64]
        L.fqro_f32_to_bf16_array.argtypes = [c_vp, c_vp, c_i64]
        L.fqro_rmsnorm.argtypes = [c_vp, c_vp, ctypes.c_int, c_f32, c_vp]
        L.fqro_rope_neox.argtypes = [c_vp, c_vp, ctypes.c_int]
        L.fqro_rope_gptj.argtypes = [c_vp, c_vp, ctypes.c_int]
        L.fqro_validate.argtypes = [c_vp, c_vp, c_i32, c_i32, c_i32, c_i32, c_i32, c_vp,
                                    c_i32, c_i32]
        L.fqro_validate.restype = ctypes.c_int
        L.fqro_append_paged.argtypes = [ctypes.POINTER(_AppendArgs)]
        L.fqro_append_paged.restype = ctypes.c_int
        L.fqro_concat_mla_cache.argtypes = [ctypes.POINTER(_MlaArgs)]
        L.fqro_concat_mla_cache.restype = ctypes.c_int
        _LIB = L
    return _LIB


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


# ---------------------------------------------------------------- formats --

def e4m3(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    lib().fqro_f32_to_e4m3_array(_ptr(x), _ptr(out), x.size)
    return out


def bf16(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().fqro_f32_to_bf16_array(_ptr(x), _ptr(out), x.size)
    return out


def bf16_to_f32(bits) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


# ------------------------------------------------------------------ steps --

def rmsnorm(x, w=None, eps=1e-6) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    w = None if w is None else np.ascontiguousarray(w, dtype=np.float32)
    y = np.empty_like(x)
    lib().fqro_rmsnorm(_ptr(x), _ptr(w), x.size, eps, _ptr(y))
    return y


def rope(y, cs_row, style: int) -> np.ndarray:
    """RoPE over the first len(cs_row) elements of y (a copy is returned)."""
    y = np.array(y, dtype=np.float32, copy=True, order="C")
    cs_row = np.ascontiguousarray(cs_row, dtype=np.float32)
    fn = lib().fqro_rope_neox if style == 0 else lib().fqro_rope_gptj
    fn(_ptr(y), _ptr(cs_row), cs_row.size)
    return y


def validate(q_indptr, seq_lens, T, max_pages, page_size, cos_sin_rows,
             positions=None, max_seqlen=0, paged=True) -> int:
    q_indptr = np.ascontiguousarray(q_indptr, dtype=np.int32)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    pos = None if positions is None else np.ascontiguousarray(positions, dtype=np.int64)
    return lib().fqro_validate(_ptr(q_indptr), _ptr(seq_lens), len(seq_lens), T,
                               max_pages, page_size, cos_sin_rows, _ptr(pos),
                               max_seqlen, 1 if paged else 0)


# ---------------------------------------------------------------- methods --

def new_outputs(w):
    """Output buffers of the append, pre-filled with sentinels (q_scale in the
    workload's layout)."""
    qdt = np.uint16 if w.quant_policy == 0 else np.uint8
    out_q = np.full((w.T, w.Hq, 128), 0xFF, dtype=qdt)
    q_scale = np.full(w.q_scale_shape, np.nan, dtype=np.float32)
    flags = np.full((w.B,), 0x5A5A5A5A, dtype=np.int32)
    return out_q, q_scale, flags


def new_kv_outputs(w):
    """Caller-owned K / V outputs [T, Hkv, 128] (cache element type),
    pre-filled with sentinels."""
    dt = np.uint16 if w.quant_policy == 0 else np.uint8
    return (np.full((w.T, w.Hkv, 128), 0xEE, dtype=dt),
            np.full((w.T, w.Hkv, 128), 0xDD, dtype=dt))


def append_paged(w, k_cache: np.ndarray, v_cache: np.ndarray, out_q: np.ndarray,
                 q_scale: Optional[np.ndarray], flags: np.ndarray, *,
                 page_table: Optional[np.ndarray] = None,
                 q_indptr: Optional[np.ndarray] = None,
                 seq_lens: Optional[np.ndarray] = None,
                 out_k: Optional[np.ndarray] = None,
                 out_v: Optional[np.ndarray] = None) -> int:
    """Run the oracle append on host caches [n_pages, page_size, Hkv, 128].

    `page_table`, `q_indptr` and `seq_lens` override the workload's arrays
    (used to remap pages into a compact host cache, or to plant malformed
    metadata).  With out_k / out_v ([T, Hkv, 128]) the K/V payloads go there
    and the caches are left alone."""
    pt = np.ascontiguousarray(w.page_table if page_table is None else page_table,
                              dtype=np.int32)
    ind = np.ascontiguousarray(w.q_indptr if q_indptr is None else q_indptr, dtype=np.int32)
    sl = np.ascontiguousarray(w.seq_lens if seq_lens is None else seq_lens, dtype=np.int32)
    qkv = np.ascontiguousarray(w.qkv)
    cs = np.ascontiguousarray(w.cos_sin)
    qw = None if w.q_norm_w is None else np.ascontiguousarray(w.q_norm_w)
    kw = None if w.k_norm_w is None else np.ascontiguousarray(w.k_norm_w)
    pos = None if w.positions is None else np.ascontiguousarray(w.positions, dtype=np.int64)
    a = _AppendArgs(
        qkv=_ptr(qkv), row_stride=w.row_stride, T=w.T, B=w.B, Hq=w.Hq, Hkv=w.Hkv,
        q_norm_w=_ptr(qw), k_norm_w=_ptr(kw), eps=w.eps,
        cos_sin=_ptr(cs), cos_sin_rows=cs.shape[0], rot_dim=w.rot_dim,
        rope_style=w.rope_style, positions=_ptr(pos),
        q_indptr=_ptr(ind), seq_lens=_ptr(sl), page_table=_ptr(pt),
        max_pages=pt.shape[1], num_pages=k_cache.shape[0], page_size=w.page_size,
        quant_policy=w.quant_policy, q_scale_inv=w.q_scale_inv,
        k_scale=w.k_scale, v_scale=w.v_scale, upper_max=w.upper_max,
        k_cache=_ptr(k_cache), v_cache=_ptr(v_cache),
        k_page_stride=int(np.prod(k_cache.shape[1:])),
        v_page_stride=int(np.prod(v_cache.shape[1:])),
        out_q=_ptr(out_q), q_scale=_ptr(q_scale), flags=_ptr(flags),
        max_seqlen=w.max_seqlen, norm_style=w.norm_style,
        out_k=_ptr(out_k), out_v=_ptr(out_v))
    return lib().fqro_append_paged(ctypes.byref(a))


def new_mla_q_outputs(w):
    """q_out [T, Hq, nope + rope] and q_scale ([T] per token, [T, Hq] per
    head) of the MLA Q quantisation, pre-filled with sentinels."""
    q_out = np.full((w.T, w.Hq, w.nope_dim + w.rope_dim), 0xFF, np.uint8)
    shape = w.q_scale_shape
    return q_out, np.full(shape, np.nan, np.float32)


def concat_mla_cache(w, q: np.ndarray, latent: np.ndarray, flags: np.ndarray, *,
                     block_table: Optional[np.ndarray] = None,
                     q_indptr: Optional[np.ndarray] = None,
                     seq_lens: Optional[np.ndarray] = None,
                     q_out: Optional[np.ndarray] = None,
                     q_scale: Optional[np.ndarray] = None) -> int:
    """Run the oracle MLA concat; q [T, Hq, nope+rope] is rotated in place (or,
    with w.q_quant, quantised into q_out / q_scale) and latent [n_blocks,
    block_size, rank + rope] receives the rows."""
    bt = np.ascontiguousarray(w.block_table if block_table is None else block_table,
                              dtype=np.int32)
    ind = np.ascontiguousarray(w.q_indptr if q_indptr is None else q_indptr, dtype=np.int32)
    sl = np.ascontiguousarray(w.seq_lens if seq_lens is None else seq_lens, dtype=np.int32)
    kv_c = np.ascontiguousarray(w.kv_c)
    k_pe = np.ascontiguousarray(w.k_pe)
    cs = np.ascontiguousarray(w.cos_sin)
    pos = None if w.positions is None else np.ascontiguousarray(w.positions, dtype=np.int64)
    assert q.flags["C_CONTIGUOUS"] and latent.flags["C_CONTIGUOUS"]
    a = _MlaArgs(
        q=_ptr(q), T=w.T, B=w.B, Hq=w.Hq, nope_dim=w.nope_dim, rope_dim=w.rope_dim,
        q_token_stride=q.shape[1] * q.shape[2], q_head_stride=q.shape[2],
        kv_c=_ptr(kv_c), kv_lora_rank=kv_c.shape[1], kv_c_stride=kv_c.shape[1],
        k_pe=_ptr(k_pe), k_pe_stride=k_pe.shape[1],
        cos_sin=_ptr(cs), cos_sin_rows=cs.shape[0], rope_style=w.rope_style,
        positions=_ptr(pos), q_indptr=_ptr(ind), seq_lens=_ptr(sl),
        block_table=_ptr(bt), max_blocks=bt.shape[1],
        latent_cache=_ptr(latent), num_blocks=latent.shape[0],
        block_size=w.block_size, cache_fp8=w.cache_fp8, kv_scale=w.kv_scale,
        flags=_ptr(flags), q_quant=w.q_quant, q_scale_inv=w.q_scale_inv,
        upper_max=w.upper_max, q_out=_ptr(q_out), q_scale=_ptr(q_scale),
        q_group=w.q_group)
    return lib().fqro_concat_mla_cache(ctypes.byref(a))


__all__ = ["lib", "e4m3", "bf16", "bf16_to_f32", "rmsnorm", "rope", "validate",
           "new_outputs", "new_kv_outputs", "new_mla_q_outputs", "append_paged",
           "concat_mla_cache"]
