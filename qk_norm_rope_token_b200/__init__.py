"""Python binding of libfqr.so (include/fqr.h): argument marshalling only.

Every step of the path runs in the library's CUDA kernels; PyTorch supplies
device memory and the stream.  There is no fallback: importing this package
fails if the library has not been built (python
qk_norm_rope_token_b200/build.py).

    append_paged(...)       -> fqr_append_paged
    append_plan(params)     -> fqr_append_plan_query (the launch, without launching)
    concat_mla_cache(...)   -> fqr_concat_mla_cache
    StagedAppend            -> fqr_pipeline_* (pinned-host batches, pipelined)

Tensors: BF16 data as torch.bfloat16 (or int16/uint16 bit patterns), FP8 E4M3
as torch.float8_e4m3fn or torch.uint8.  All on one CUDA device.
"""
from __future__ import annotations

import ctypes

import numpy as np
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfqr.so")

FQR_OK, FQR_EINVAL, FQR_ENOTSUP, FQR_ECUDA = 0, 1, 2, 3
SCHEDULE_AUTO, SCHEDULE_LATENCY, SCHEDULE_STREAMING = 0, 1, 2
FLAG_TIMEOUT = -2
NORM_RMS, NORM_GEMMA = 0, 1
MLA_Q_NONE, MLA_Q_STATIC, MLA_Q_TOKEN, MLA_Q_HEAD, MLA_Q_GROUP = 0, 1, 2, 3, 4
HEAD_DIM = 128
MAX_BATCH = 16384

c_i32, c_i64, c_f32, c_vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p


class AppendParams(ctypes.Structure):
    """Mirror of fqr_append_params."""
    _fields_ = [
        ("qkv", c_vp), ("qkv_row_stride", c_i64),
        ("T", c_i32), ("B", c_i32), ("Hq", c_i32), ("Hkv", c_i32), ("head_dim", c_i32),
        ("q_norm_w", c_vp), ("k_norm_w", c_vp), ("eps", c_f32),
        ("cos_sin_cache", c_vp), ("cos_sin_rows", c_i32), ("rot_dim", c_i32),
        ("rope_style", c_i32), ("positions", c_vp),
        ("q_indptr", c_vp), ("seq_lens", c_vp), ("page_table", c_vp), ("max_pages", c_i32),
        ("k_cache", c_vp), ("v_cache", c_vp), ("num_pages", c_i32), ("page_size", c_i32),
        ("k_page_stride", c_i64), ("v_page_stride", c_i64),
        ("quant_policy", c_i32),
        ("q_scale_inv", c_vp), ("k_scale", c_vp), ("v_scale", c_vp), ("upper_max", c_f32),
        ("out_q", c_vp), ("q_scale", c_vp), ("flags", c_vp), ("schedule", c_i32),
        ("max_seqlen", c_i32), ("norm_style", c_i32), ("out_k", c_vp), ("out_v", c_vp),
    ]


class AppendPlan(ctypes.Structure):
    """Mirror of fqr_append_plan."""
    _fields_ = [("schedule", c_i32), ("grid", c_i32), ("block_threads", c_i32), ("tasks", c_i32),
                ("warp_check", c_i32), ("bulk_tails", c_i32), ("request_tails", c_i32)]


class MlaParams(ctypes.Structure):
    """Mirror of fqr_mla_params."""
    _fields_ = [
        ("q", c_vp), ("T", c_i32), ("B", c_i32), ("Hq", c_i32), ("nope_dim", c_i32),
        ("rope_dim", c_i32), ("q_token_stride", c_i64), ("q_head_stride", c_i64),
        ("kv_c", c_vp), ("kv_lora_rank", c_i32), ("kv_c_stride", c_i64),
        ("k_pe", c_vp), ("k_pe_stride", c_i64),
        ("cos_sin_cache", c_vp), ("cos_sin_rows", c_i32), ("rope_style", c_i32),
        ("positions", c_vp), ("q_indptr", c_vp), ("seq_lens", c_vp),
        ("block_table", c_vp), ("max_blocks", c_i32),
        ("latent_cache", c_vp), ("num_blocks", c_i32), ("block_size", c_i32),
        ("cache_fp8", c_i32), ("kv_scale", c_vp), ("flags", c_vp),
        ("q_quant", c_i32), ("q_scale_inv", c_vp), ("upper_max", c_f32),
        ("q_out", c_vp), ("q_scale", c_vp), ("q_group", c_i32),
    ]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python qk_norm_rope_token_b200/build.py` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    lib.fqr_append_paged.argtypes = [ctypes.POINTER(AppendParams), c_vp]
    lib.fqr_append_paged.restype = ctypes.c_int
    lib.fqr_concat_mla_cache.argtypes = [ctypes.POINTER(MlaParams), c_vp]
    lib.fqr_concat_mla_cache.restype = ctypes.c_int
    lib.fqr_append_plan_query.argtypes = [ctypes.POINTER(AppendParams),
                                          ctypes.POINTER(AppendPlan)]
    lib.fqr_append_plan_query.restype = ctypes.c_int
    lib.fqr_strerror.argtypes = [ctypes.c_int]
    lib.fqr_strerror.restype = ctypes.c_char_p
    lib.fqr_pipeline_create.argtypes = [ctypes.c_int, ctypes.POINTER(AppendParams),
                                        ctypes.POINTER(c_vp), ctypes.c_size_t,
                                        ctypes.POINTER(c_vp), ctypes.c_size_t,
                                        ctypes.POINTER(c_vp)]
    for name in ("fqr_pipeline_create", "fqr_pipeline_submit", "fqr_pipeline_fork",
                 "fqr_pipeline_join", "fqr_pipeline_sync", "fqr_pipeline_destroy"):
        getattr(lib, name).restype = ctypes.c_int
    lib.fqr_pipeline_submit.argtypes = [c_vp, c_vp, c_vp]
    lib.fqr_pipeline_fork.argtypes = [c_vp, c_vp]
    lib.fqr_pipeline_join.argtypes = [c_vp, c_vp]
    lib.fqr_pipeline_sync.argtypes = [c_vp]
    lib.fqr_pipeline_destroy.argtypes = [c_vp]
    return lib


LIB = _load()


class FqrError(RuntimeError):
    def __init__(self, code: int):
        self.code = code
        super().__init__(f"fqr error {code}: {LIB.fqr_strerror(code).decode()}")


def strerror(code: int) -> str:
    return LIB.fqr_strerror(code).decode()


def append_paged_raw(params: AppendParams, stream: int = 0) -> int:
    """Call fqr_append_paged with a filled parameter struct; returns the code."""
    return LIB.fqr_append_paged(ctypes.byref(params), c_vp(stream))


def append_plan(params: AppendParams) -> dict:
    """fqr_append_plan_query: the launch fqr_append_paged would make for these
    parameters on the current device (nothing is launched).  Raises FqrError
    on a rejected argument."""
    plan = AppendPlan()
    rc = LIB.fqr_append_plan_query(ctypes.byref(params), ctypes.byref(plan))
    if rc != FQR_OK:
        raise FqrError(rc)
    return {name: int(getattr(plan, name)) for name, _ in AppendPlan._fields_}


def concat_mla_cache_raw(params: MlaParams, stream: int = 0) -> int:
    return LIB.fqr_concat_mla_cache(ctypes.byref(params), c_vp(stream))


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream, device) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def append_params(qkv, cos_sin_cache, q_indptr, seq_lens, page_table, k_cache, v_cache,
                  out_q, flags, *, q_norm_w=None, k_norm_w=None, eps: float = 1e-6,
                  positions=None, rope_style: int = 0, rot_dim: Optional[int] = None,
                  quant_policy: int = 0, q_scale=None, q_scale_inv=None, k_scale=None,
                  v_scale=None, upper_max: float = 448.0,
                  schedule: int = SCHEDULE_AUTO, max_seqlen: int = 0,
                  norm_style: int = NORM_RMS, out_k=None, out_v=None) -> AppendParams:
    """Fill an AppendParams from tensors (shapes as in include/fqr.h).  With
    out_k / out_v ([T, Hkv, 128]) the K/V payloads go there; k_cache, v_cache
    and page_table may then be None."""
    T = int(qkv.shape[0])
    kv = k_cache if k_cache is not None else out_k
    paged = k_cache is not None
    return AppendParams(
        qkv=_ptr(qkv), qkv_row_stride=int(qkv.stride(0)) if T > 0 else int(qkv.shape[1]),
        T=T, B=int(seq_lens.numel()), Hq=int(out_q.shape[1]), Hkv=int(kv.shape[-2]),
        head_dim=int(kv.shape[-1]),
        q_norm_w=_ptr(q_norm_w), k_norm_w=_ptr(k_norm_w), eps=float(eps),
        cos_sin_cache=_ptr(cos_sin_cache), cos_sin_rows=int(cos_sin_cache.shape[0]),
        rot_dim=int(cos_sin_cache.shape[1] if rot_dim is None else rot_dim),
        rope_style=int(rope_style), positions=_ptr(positions),
        q_indptr=_ptr(q_indptr), seq_lens=_ptr(seq_lens), page_table=_ptr(page_table),
        max_pages=int(page_table.shape[1]) if page_table is not None else 0,
        k_cache=_ptr(k_cache), v_cache=_ptr(v_cache),
        num_pages=int(k_cache.shape[0]) if paged else 0,
        page_size=int(k_cache.shape[1]) if paged else 0,
        k_page_stride=int(k_cache.stride(0)) if paged else 0,
        v_page_stride=int(v_cache.stride(0)) if paged else 0,
        quant_policy=int(quant_policy), q_scale_inv=_ptr(q_scale_inv),
        k_scale=_ptr(k_scale), v_scale=_ptr(v_scale), upper_max=float(upper_max),
        out_q=_ptr(out_q), q_scale=_ptr(q_scale), flags=_ptr(flags), schedule=int(schedule),
        max_seqlen=int(max_seqlen), norm_style=int(norm_style),
        out_k=_ptr(out_k), out_v=_ptr(out_v))


def append_paged(qkv, cos_sin_cache, q_indptr, seq_lens, page_table, k_cache, v_cache,
                 out_q, flags, *, stream=None, **kw) -> None:
    """Fused QK RMSNorm + RoPE + (FP8) quantisation + paged KV append.

    qkv [T, >= (Hq+2Hkv)*128] bf16 (unit inner stride), cos_sin_cache
    [rows, rot] fp32, q_indptr [B+1] / seq_lens [B] int32, page_table
    [B, max_pages] int32, k_cache / v_cache [num_pages, page_size, Hkv, 128],
    out_q [T, Hq, 128], flags [B] int32; keyword arguments as in
    append_params.  Enqueued on `stream` (default: torch's current stream).
    Raises FqrError on a host-side argument error."""
    p = append_params(qkv, cos_sin_cache, q_indptr, seq_lens, page_table, k_cache, v_cache,
                      out_q, flags, **kw)
    rc = append_paged_raw(p, _stream(stream, qkv.device))
    if rc != FQR_OK:
        raise FqrError(rc)


def append_paged_from_host(host_in: dict, dev_in: dict, host_out: dict, dev_out: dict, *,
                           cos_sin_cache, k_cache, v_cache, stream=None, **kw) -> None:
    """append_paged with the step's inputs and results in (pinned) host memory.

    host_in / dev_in map "qkv", "q_indptr", "seq_lens", "page_table" (and
    optionally "positions") to host tensors and same-shaped device staging
    tensors; host_out / dev_out map "out_q", "flags" (and "q_scale" for the
    dynamic policy) likewise.  Enqueues, on one stream: the host-to-device
    copies, the fused kernel, and the device-to-host copies of the results.
    The KV caches, the cos/sin cache and the norm weights stay resident on the
    device.  The caller synchronises before reading host_out."""
    import torch
    s = torch.cuda.current_stream(k_cache.device) if stream is None else stream
    with torch.cuda.stream(s):
        for k, h in host_in.items():
            dev_in[k].copy_(h, non_blocking=True)
        extra = {"positions": dev_in["positions"]} if "positions" in dev_in else {}
        if "q_scale" in dev_out:
            extra["q_scale"] = dev_out["q_scale"]
        append_paged(dev_in["qkv"], cos_sin_cache, dev_in["q_indptr"], dev_in["seq_lens"],
                     dev_in["page_table"], k_cache, v_cache, dev_out["out_q"], dev_out["flags"],
                     stream=s, **extra, **kw)
        for k, h in host_out.items():
            h.copy_(dev_out[k], non_blocking=True)


class StagedAppend:
    """append_paged on batches that live in pinned host memory, pipelined by
    the library's native pipeline (fqr_pipeline_* in include/fqr.h).

    Each submit() enqueues, for one batch: the host-to-device copy of its
    inputs, the fused kernel and the device-to-host copy of its results, on
    three streams with events between them and `depth` sets of device staging
    buffers rotated.  So the copy-in of the next batch, the kernel of this one
    and the copy-out of the previous one overlap (PCIe carries both directions
    at once).

    in_shapes / out_shapes map the names of append_paged_from_host ("qkv",
    "q_indptr", "seq_lens", "page_table", optionally "positions"; "out_q",
    "flags", optionally "q_scale") to (shape, dtype).  Each slot's inputs (and
    results) are views of one flat device buffer; new_host_buffers() returns
    matching pinned host views of one flat buffer each way, so a batch moves
    in one copy each way.  The KV caches, cos/sin cache, norm weights and the
    other append_paged keywords are fixed at construction.  synchronize()
    waits for every submitted batch; join(stream) makes a stream wait for
    them."""

    _ALIGN = 256

    def __init__(self, in_shapes: dict, out_shapes: dict, device, depth: int = 2, *,
                 cos_sin_cache, k_cache, v_cache, **kw):
        import torch
        self.torch = torch
        self.depth = depth
        self.in_shapes, self.out_shapes = dict(in_shapes), dict(out_shapes)
        self.in_bytes, self.in_offs = self._layout(self.in_shapes)
        self.out_bytes, self.out_offs = self._layout(self.out_shapes)
        self.flat_in = [torch.empty(self.in_bytes, dtype=torch.uint8, device=device) for _ in range(depth)]
        self.flat_out = [torch.empty(self.out_bytes, dtype=torch.uint8, device=device)
                         for _ in range(depth)]
        self.dev_in = [self._views(f, self.in_shapes, self.in_offs) for f in self.flat_in]
        self.dev_out = [self._views(f, self.out_shapes, self.out_offs) for f in self.flat_out]
        params = []
        for din, dout in zip(self.dev_in, self.dev_out):
            extra = {"positions": din["positions"]} if "positions" in din else {}
            if "q_scale" in dout:
                extra["q_scale"] = dout["q_scale"]
            params.append(append_params(din["qkv"], cos_sin_cache, din["q_indptr"],
                                        din["seq_lens"], din["page_table"], k_cache, v_cache,
                                        dout["out_q"], dout["flags"], **extra, **kw))
        self._keep = (cos_sin_cache, k_cache, v_cache, kw)
        self._params = (AppendParams * depth)(*params)
        dev_in = (c_vp * depth)(*[f.data_ptr() for f in self.flat_in])
        dev_out = (c_vp * depth)(*[f.data_ptr() for f in self.flat_out])
        self._handle = c_vp()
        rc = LIB.fqr_pipeline_create(depth, self._params, dev_in, self.in_bytes, dev_out,
                                     self.out_bytes, ctypes.byref(self._handle))
        if rc != FQR_OK:
            self._handle = None
            raise FqrError(rc)

    @classmethod
    def _layout(cls, shapes):
        import torch
        offs, n = {}, 0
        for k, (sh, dt) in shapes.items():
            offs[k] = n
            size = int(np.prod(sh)) * torch.empty((), dtype=dt).element_size()
            n += -(-size // cls._ALIGN) * cls._ALIGN
        return max(n, cls._ALIGN), offs

    @staticmethod
    def _views(flat, shapes, offs):
        import torch
        out = {}
        for k, (sh, dt) in shapes.items():
            size = int(np.prod(sh)) * torch.empty((), dtype=dt).element_size()
            out[k] = flat[offs[k]:offs[k] + size].view(dt).view(sh)
        return out

    def new_host_buffers(self):
        """(host_in, host_out): pinned host views, each set backed by one flat
        buffer (kept under the key "_flat")."""
        torch = self.torch
        fin = torch.empty(self.in_bytes, dtype=torch.uint8).pin_memory()
        fout = torch.empty(self.out_bytes, dtype=torch.uint8).pin_memory()
        hin = self._views(fin, self.in_shapes, self.in_offs)
        hout = self._views(fout, self.out_shapes, self.out_offs)
        hin["_flat"], hout["_flat"] = fin, fout
        return hin, hout

    def submit(self, host_in: dict, host_out: dict) -> None:
        """Enqueue one batch (buffers from new_host_buffers)."""
        rc = LIB.fqr_pipeline_submit(self._handle, c_vp(host_in["_flat"].data_ptr()),
                                     c_vp(host_out["_flat"].data_ptr()))
        if rc != FQR_OK:
            raise FqrError(rc)

    def fork(self, stream) -> None:
        """The pipeline's streams wait for the work enqueued so far on `stream`."""
        rc = LIB.fqr_pipeline_fork(self._handle, c_vp(_stream(stream, None)))
        if rc != FQR_OK:
            raise FqrError(rc)

    def join(self, stream) -> None:
        """`stream` waits for every batch submitted so far."""
        rc = LIB.fqr_pipeline_join(self._handle, c_vp(_stream(stream, None)))
        if rc != FQR_OK:
            raise FqrError(rc)

    def synchronize(self) -> None:
        rc = LIB.fqr_pipeline_sync(self._handle)
        if rc != FQR_OK:
            raise FqrError(rc)

    def close(self) -> None:
        if self._handle:
            LIB.fqr_pipeline_destroy(self._handle)
            self._handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def mla_params(q, kv_c, k_pe, cos_sin_cache, q_indptr, seq_lens, block_table, latent_cache,
               flags, *, nope_dim: int, rope_style: int = 1, kv_scale=None,
               positions=None, q_quant: int = MLA_Q_NONE, q_scale_inv=None,
               upper_max: float = 448.0, q_out=None, q_scale=None,
               q_group: int = 0) -> MlaParams:
    T = int(q.shape[0])
    rope_dim = int(k_pe.shape[1]) if k_pe.dim() == 2 else 0
    return MlaParams(
        q=_ptr(q), T=T, B=int(seq_lens.numel()), Hq=int(q.shape[1]), nope_dim=int(nope_dim),
        rope_dim=rope_dim, q_token_stride=int(q.stride(0)), q_head_stride=int(q.stride(1)),
        kv_c=_ptr(kv_c), kv_lora_rank=int(kv_c.shape[1]), kv_c_stride=int(kv_c.stride(0)),
        k_pe=_ptr(k_pe), k_pe_stride=int(k_pe.stride(0)),
        cos_sin_cache=_ptr(cos_sin_cache), cos_sin_rows=int(cos_sin_cache.shape[0]),
        rope_style=int(rope_style), positions=_ptr(positions),
        q_indptr=_ptr(q_indptr), seq_lens=_ptr(seq_lens), block_table=_ptr(block_table),
        max_blocks=int(block_table.shape[1]), latent_cache=_ptr(latent_cache),
        num_blocks=int(latent_cache.shape[0]), block_size=int(latent_cache.shape[1]),
        cache_fp8=1 if latent_cache.element_size() == 1 else 0, kv_scale=_ptr(kv_scale),
        flags=_ptr(flags), q_quant=int(q_quant), q_scale_inv=_ptr(q_scale_inv),
        upper_max=float(upper_max), q_out=_ptr(q_out), q_scale=_ptr(q_scale),
        q_group=int(q_group))


def concat_mla_cache(q, kv_c, k_pe, cos_sin_cache, q_indptr, seq_lens, block_table,
                     latent_cache, flags, *, stream=None, **kw) -> None:
    """MLA: rotate q[..., nope:nope+64] in place (or, with q_quant, quantise
    [nope | rope(rope part)] into q_out / q_scale) and write [kv_c |
    rope(k_pe)] rows into latent_cache [num_blocks, block_size, rank + 64]
    (e4m3 with *kv_scale, or bf16).  Raises FqrError on a host-side argument
    error."""
    p = mla_params(q, kv_c, k_pe, cos_sin_cache, q_indptr, seq_lens, block_table,
                   latent_cache, flags, **kw)
    rc = concat_mla_cache_raw(p, _stream(stream, latent_cache.device))
    if rc != FQR_OK:
        raise FqrError(rc)


__all__ = ["LIB", "LIB_PATH", "AppendParams", "MlaParams", "FqrError", "strerror",
           "append_paged_from_host", "StagedAppend",
           "append_params", "append_paged", "append_paged_raw", "mla_params",
           "concat_mla_cache", "concat_mla_cache_raw", "FQR_OK", "FQR_EINVAL",
           "FQR_ENOTSUP", "FQR_ECUDA", "HEAD_DIM", "MAX_BATCH", "SCHEDULE_AUTO",
           "SCHEDULE_LATENCY", "SCHEDULE_STREAMING", "FLAG_TIMEOUT", "NORM_RMS",
           "NORM_GEMMA", "MLA_Q_NONE", "MLA_Q_STATIC", "MLA_Q_TOKEN", "MLA_Q_HEAD",
           "MLA_Q_GROUP"]
