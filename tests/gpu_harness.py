"""GPU-vs-oracle parity harness for the paged append and the MLA concat.

The CUDA path runs through the C ABI (the Python binding) on device tensors;
the oracle runs on host copies of exactly the same inputs.  The caches can be
GiBs, so the oracle gets a COMPACT cache holding only the pages the call may
touch (the pages of the new tokens' positions and each request's last page),
remapped through the page table; every other page is checked on the device to
be byte-identical to its pre-call content.

Bars (from the method's tolerance statement): bitwise for slots, flags,
untouched bytes, zero tails and V copies; <= 1 BF16 ulp for BF16 results;
<= 1 E4M3 ulp for FP8 payloads; q_scale relative error <= 1e-5.  check()
asserts these on every element and reports the fraction of payloads and
scales that are bit-identical; tests that expect bit-identical results (both
sides evaluate the same correctly rounded steps) assert that on the report.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import qk_norm_rope_token_b200 as fqr
from tests._util import ulp_bf16, ulp_e4m3

D = 128
DEV = "cuda"


def _dt(esize):
    return torch.int16 if esize == 2 else torch.uint8


def _np(t):
    a = t.cpu().numpy()
    return a.view(np.uint16) if a.dtype == np.int16 else a


def _dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if t.dtype == torch.uint16:
        t = t.view(torch.int16)
    if dtype is not None:
        t = t.to(dtype)
    return t.to(DEV)


def fill_random_(t: torch.Tensor, seed: int):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    flat = t.view(torch.uint8).view(-1)
    step = 1 << 28
    for i in range(0, flat.numel(), step):
        n = min(step, flat.numel() - i)
        flat[i:i + n] = torch.randint(0, 256, (n,), dtype=torch.uint8, device=DEV, generator=g)


def touched_pages(page_table, q_indptr, seq_lens, P):
    pages = set()
    for b in range(len(seq_lens)):
        lo, hi, L = int(q_indptr[b]), int(q_indptr[b + 1]), int(seq_lens[b])
        for p in range(L - (hi - lo), L):
            pages.add(int(page_table[b, p // P]))
        if L > 0:
            pages.add(int(page_table[b, (L - 1) // P]))
    return sorted(pages)


def changed_pages(after: torch.Tensor, before: torch.Tensor, chunk=2048) -> set:
    a = after.view(after.shape[0], -1).view(torch.uint8)
    b = before.view(before.shape[0], -1).view(torch.uint8)
    out = []
    for i in range(0, a.shape[0], chunk):
        d = (a[i:i + chunk] != b[i:i + chunk]).any(dim=1)
        out.append(torch.nonzero(d).flatten() + i)
    return set(torch.cat(out).tolist()) if out else set()


class AppendRun:
    """Device state of one fqr_append_paged call plus what the oracle needs."""

    def __init__(self, w, *, fill_seed=11, q_indptr=None, seq_lens=None, page_stride_pad=0,
                 schedule=0, null_caches=True):
        self.w = w
        self.schedule = schedule
        self.owned = bool(w.out_kv)
        # with caller-owned K/V the caches and the page table are passed as NULL
        # (unless null_caches is False); the caches still exist here so that
        # every byte of them can be checked to be untouched
        self.null_caches = self.owned and null_caches
        self.q_indptr = np.asarray(w.q_indptr if q_indptr is None else q_indptr, np.int32)
        self.seq_lens = np.asarray(w.seq_lens if seq_lens is None else seq_lens, np.int32)
        es = w.kv_esize
        P = w.page_size
        self.qkv = _dev(w.qkv)
        self.cs = _dev(w.cos_sin)
        self.indptr_d = _dev(self.q_indptr)
        self.seq_d = _dev(self.seq_lens)
        self.pt_d = _dev(w.page_table)
        self.pos_d = None if w.positions is None else _dev(w.positions)
        self.qw = None if w.q_norm_w is None else _dev(w.q_norm_w)
        self.kw = None if w.k_norm_w is None else _dev(w.k_norm_w)
        # caches, optionally with padded page strides
        inner = P * w.Hkv * D
        stride = inner + page_stride_pad
        self.k_store = torch.empty((w.num_pages, stride), dtype=_dt(es), device=DEV)
        self.v_store = torch.empty((w.num_pages, stride), dtype=_dt(es), device=DEV)
        fill_random_(self.k_store, fill_seed)
        fill_random_(self.v_store, fill_seed + 1)
        self.k_cache = self.k_store[:, :inner].view(w.num_pages, P, w.Hkv, D) if page_stride_pad == 0 \
            else torch.as_strided(self.k_store, (w.num_pages, P, w.Hkv, D), (stride, w.Hkv * D, D, 1))
        self.v_cache = self.v_store[:, :inner].view(w.num_pages, P, w.Hkv, D) if page_stride_pad == 0 \
            else torch.as_strided(self.v_store, (w.num_pages, P, w.Hkv, D), (stride, w.Hkv * D, D, 1))
        self.k_before = self.k_store.clone()
        self.v_before = self.v_store.clone()
        self.out_q = torch.empty((w.T, w.Hq, D), dtype=_dt(w.q_esize), device=DEV)
        fill_random_(self.out_q, fill_seed + 2)
        self.out_q_before = self.out_q.clone()
        qs_shape = w.q_scale_shape if w.max_seqlen > 0 or w.T > 0 else (1, w.Hq)
        self.q_scale = torch.full(qs_shape, float("nan"), device=DEV)
        self.q_scale_before = self.q_scale.clone()
        if self.owned:
            self.out_k = torch.empty((w.T, w.Hkv, D), dtype=_dt(es), device=DEV)
            self.out_v = torch.empty((w.T, w.Hkv, D), dtype=_dt(es), device=DEV)
            fill_random_(self.out_k, fill_seed + 3)
            fill_random_(self.out_v, fill_seed + 4)
            self.out_k_before = self.out_k.clone()
            self.out_v_before = self.out_v.clone()
        self.flags = torch.full((w.B,), 0x5A5A5A5A, dtype=torch.int32, device=DEV)
        self.scales = {k: torch.tensor([v], dtype=torch.float32, device=DEV)
                       for k, v in (("q_scale_inv", w.q_scale_inv), ("k_scale", w.k_scale),
                                    ("v_scale", w.v_scale))}

    def kwargs(self):
        w = self.w
        return dict(q_norm_w=self.qw, k_norm_w=self.kw, eps=w.eps, positions=self.pos_d,
                    rope_style=w.rope_style, rot_dim=w.rot_dim, quant_policy=w.quant_policy,
                    q_scale=self.q_scale if w.quant_policy == 1 else None,
                    q_scale_inv=self.scales["q_scale_inv"] if w.quant_policy == 2 else None,
                    k_scale=self.scales["k_scale"] if w.quant_policy else None,
                    v_scale=self.scales["v_scale"] if w.quant_policy else None,
                    upper_max=w.upper_max, schedule=self.schedule, max_seqlen=w.max_seqlen,
                    norm_style=w.norm_style,
                    out_k=self.out_k if self.owned else None,
                    out_v=self.out_v if self.owned else None)

    def launch(self, stream=None):
        nul = self.null_caches
        fqr.append_paged(self.qkv, self.cs, self.indptr_d, self.seq_d,
                         None if nul else self.pt_d, None if nul else self.k_cache,
                         None if nul else self.v_cache, self.out_q, self.flags, stream=stream,
                         **self.kwargs())

    def plan(self):
        """The launch plan of this call (fqr_append_plan_query)."""
        nul = self.null_caches
        return fqr.append_plan(fqr.append_params(
            self.qkv, self.cs, self.indptr_d, self.seq_d, None if nul else self.pt_d,
            None if nul else self.k_cache, None if nul else self.v_cache, self.out_q, self.flags,
            **self.kwargs()))

    # ------------------------------------------------------------ checking --
    def run_oracle(self):
        w = self.w
        P = w.page_size
        valid = oracle.validate(self.q_indptr, self.seq_lens, w.T, w.max_pages, P,
                                w.cos_sin_rows, w.positions,
                                max_seqlen=w.max_seqlen if w.quant_policy == 1 else 0,
                                paged=not self.owned) == 0
        pages = touched_pages(w.page_table, self.q_indptr, self.seq_lens, P) \
            if valid and not self.owned else []
        remap = {g: i for i, g in enumerate(pages)}
        pt = np.full_like(w.page_table, -1)
        for (b, k), g in np.ndenumerate(w.page_table):
            if int(g) in remap:
                pt[b, k] = remap[int(g)]
        idx = torch.tensor(pages, dtype=torch.long, device=DEV)
        inner = P * w.Hkv * D
        shape = (len(pages), P, w.Hkv, D)
        kc = _np(self.k_before[idx, :inner]).reshape(shape).copy() if pages else \
            np.zeros((1, P, w.Hkv, D), _np(self.k_before[:1]).dtype)
        vc = _np(self.v_before[idx, :inner]).reshape(shape).copy() if pages else kc.copy()
        oq = _np(self.out_q_before).copy()
        qs = self.q_scale_before.cpu().numpy().copy()
        fl = np.full(w.B, 0x5A5A5A5A, np.int32)
        ok = _np(self.out_k_before).copy() if self.owned else None
        ov = _np(self.out_v_before).copy() if self.owned else None
        rc = oracle.append_paged(w, kc, vc, oq, qs if w.quant_policy == 1 else None, fl,
                                 page_table=pt, q_indptr=self.q_indptr, seq_lens=self.seq_lens,
                                 out_k=ok, out_v=ov)
        return dict(rc=rc, pages=pages, idx=idx, k=kc, v=vc, out_q=oq, q_scale=qs, flags=fl,
                    out_k=ok, out_v=ov)

    def q_scale_at(self, qs, r, h):
        """q_scale of packed row r, Q head h, in the call's layout."""
        if self.w.max_seqlen > 0:
            b = int(np.searchsorted(self.q_indptr, r, side="right") - 1)
            return float(qs[b, h, r - int(self.q_indptr[b])])
        return float(qs[r, h])

    def check(self, ref=None):
        """Compare the device state with the oracle; returns a small report."""
        w = self.w
        ref = self.run_oracle() if ref is None else ref
        rep = {}
        torch.cuda.synchronize()
        # flags bitwise
        assert np.array_equal(self.flags.cpu().numpy(), ref["flags"]), "flags"
        # inputs untouched
        assert np.array_equal(_np(self.qkv), w.qkv), "qkv (incl. V and padding) modified"
        # pages outside the touched set: byte-identical
        touched = set(ref["pages"])
        for name, after, before in (("k", self.k_store, self.k_before),
                                    ("v", self.v_store, self.v_before)):
            extra = changed_pages(after, before) - touched
            assert not extra, f"{name} cache: untouched pages written: {sorted(extra)[:8]}"
        if self.owned:
            assert not changed_pages(self.k_store, self.k_before), "k cache written (owned K/V)"
            assert not changed_pages(self.v_store, self.v_before), "v cache written (owned K/V)"
        if ref["rc"] != 0:   # malformed: nothing but the flags may change
            assert torch.equal(self.out_q, self.out_q_before), "out_q written on a flagged call"
            if w.quant_policy == 1:
                assert torch.isnan(self.q_scale).all(), "q_scale written on a flagged call"
            if self.owned:
                assert torch.equal(self.out_k, self.out_k_before), "out_k written on a flagged call"
                assert torch.equal(self.out_v, self.out_v_before), "out_v written on a flagged call"
            return {"flagged": True}
        if self.owned and w.T:
            og, ovg = _np(self.out_k), _np(self.out_v)
            assert np.array_equal(ovg, ref["out_v"]), "owned V rows"
            ulp = ulp_bf16 if w.kv_esize == 2 else ulp_e4m3
            d = ulp(og, ref["out_k"])
            assert d.max() <= 1, f"owned K: max ulp {d.max()}"
            rep["k_exact_frac"] = float((d == 0).mean())
        # touched pages
        inner = w.page_size * w.Hkv * D
        shape = (len(ref["pages"]),) + tuple(self.k_cache.shape[1:])
        if ref["pages"]:
            kg = _np(self.k_store[ref["idx"], :inner]).reshape(shape)
            vg = _np(self.v_store[ref["idx"], :inner]).reshape(shape)
            assert np.array_equal(vg, ref["v"]), "V rows / tails / untouched V bytes"
            kmask = self._k_written_rows(ref)
            assert np.array_equal(kg[~kmask], ref["k"][~kmask]), "K tails / untouched K bytes"
            ulp = ulp_bf16 if w.kv_esize == 2 else ulp_e4m3
            d = ulp(kg, ref["k"])
            d = np.where(kmask, d, 0)
            assert d.max() <= 1, f"K rows: max ulp {d.max()}"
            rep["k_exact_frac"] = float((d[kmask] == 0).mean()) if kmask.any() else 1.0
        # out_q
        oq = _np(self.out_q)
        if w.T:
            d = (ulp_bf16 if w.q_esize == 2 else ulp_e4m3)(oq, ref["out_q"])
            assert d.max() <= 1, f"out_q: max ulp {d.max()}"
            rep["q_exact_frac"] = float((d == 0).mean())
            if w.quant_policy == 1:
                qs = self.q_scale.cpu().numpy()
                want = ref["q_scale"]
                # entries no token owns (prefill padding) stay untouched
                assert np.array_equal(np.isnan(qs), np.isnan(want)), "q_scale entries written"
                m = ~np.isnan(want)
                rel = np.abs(qs[m] - want[m]) / np.abs(want[m])
                assert rel.max() <= 1e-5, f"q_scale rel {rel.max()}"
                rep["q_scale_rel_max"] = float(rel.max())
                rep["q_scale_exact_frac"] = float(
                    (qs[m].view(np.uint32) == want[m].view(np.uint32)).mean())
        return rep

    def _k_written_rows(self, ref):
        """bool mask over the compact K image: rows written by new tokens."""
        w = self.w
        P = w.page_size
        remap = {g: i for i, g in enumerate(ref["pages"])}
        mask = np.zeros(ref["k"].shape, bool)
        for b in range(w.B):
            lo, hi, L = int(self.q_indptr[b]), int(self.q_indptr[b + 1]), int(self.seq_lens[b])
            for p in range(L - (hi - lo), L):
                mask[remap[int(w.page_table[b, p // P])], p % P] = True
        return mask


class MlaRun:
    def __init__(self, w, *, fill_seed=21, q_indptr=None, seq_lens=None):
        self.w = w
        self.q_indptr = np.asarray(w.q_indptr if q_indptr is None else q_indptr, np.int32)
        self.seq_lens = np.asarray(w.seq_lens if seq_lens is None else seq_lens, np.int32)
        self.q = _dev(w.q)
        self.kv_c = _dev(w.kv_c)
        self.k_pe = _dev(w.k_pe)
        self.cs = _dev(w.cos_sin)
        self.indptr_d = _dev(self.q_indptr)
        self.seq_d = _dev(self.seq_lens)
        self.bt_d = _dev(w.block_table)
        self.pos_d = None if w.positions is None else _dev(w.positions)
        es = 1 if w.cache_fp8 else 2
        self.latent = torch.empty((w.num_blocks, w.block_size, w.width), dtype=_dt(es),
                                  device=DEV)
        fill_random_(self.latent, fill_seed)
        self.latent_before = self.latent.clone()
        self.flags = torch.full((w.B,), 0x5A5A5A5A, dtype=torch.int32, device=DEV)
        self.kv_scale = torch.tensor([w.kv_scale], dtype=torch.float32, device=DEV)
        self.qq = {}
        if w.q_quant:   # quantised Q: q_out codes and q_scale, sentinel-filled
            q_out, q_scale = oracle.new_mla_q_outputs(w)
            self.q_out = torch.empty(q_out.shape, dtype=torch.uint8, device=DEV)
            fill_random_(self.q_out, fill_seed + 5)
            self.q_out_before = self.q_out.clone()
            self.q_scale = torch.from_numpy(q_scale).to(DEV)
            self.qsi = torch.tensor([w.q_scale_inv], dtype=torch.float32, device=DEV)
            self.qq = dict(q_quant=w.q_quant, q_scale_inv=self.qsi, upper_max=w.upper_max,
                           q_out=self.q_out, q_scale=self.q_scale, q_group=w.q_group)

    def launch(self, stream=None):
        fqr.concat_mla_cache(self.q, self.kv_c, self.k_pe, self.cs, self.indptr_d, self.seq_d,
                             self.bt_d, self.latent, self.flags, nope_dim=self.w.nope_dim,
                             rope_style=self.w.rope_style, kv_scale=self.kv_scale,
                             positions=self.pos_d, stream=stream, **self.qq)

    def check(self):
        w = self.w
        bs = w.block_size
        valid = oracle.validate(self.q_indptr, self.seq_lens, w.T, w.max_blocks, bs,
                                w.cos_sin_rows, w.positions) == 0
        blocks = []
        if valid:
            for b in range(w.B):
                lo, hi, L = int(self.q_indptr[b]), int(self.q_indptr[b + 1]), int(self.seq_lens[b])
                for p in range(L - (hi - lo), L):
                    blocks.append(int(w.block_table[b, p // bs]))
        blocks = sorted(set(blocks))
        remap = {g: i for i, g in enumerate(blocks)}
        bt = np.full_like(w.block_table, -1)
        for (b, k), g in np.ndenumerate(w.block_table):
            if int(g) in remap:
                bt[b, k] = remap[int(g)]
        idx = torch.tensor(blocks, dtype=torch.long, device=DEV)
        lat = _np(self.latent_before[idx]).copy() if blocks else \
            np.zeros((1, bs, w.width), _np(self.latent_before[:1]).dtype)
        q = w.q.copy()
        fl = np.full(w.B, 0x5A5A5A5A, np.int32)
        qo = _np(self.q_out_before).copy() if w.q_quant else None
        qs = oracle.new_mla_q_outputs(w)[1] if w.q_quant else None
        rc = oracle.concat_mla_cache(w, q, lat, fl, block_table=bt, q_indptr=self.q_indptr,
                                     seq_lens=self.seq_lens, q_out=qo, q_scale=qs)
        torch.cuda.synchronize()
        assert np.array_equal(self.flags.cpu().numpy(), fl), "flags"
        assert np.array_equal(_np(self.kv_c), w.kv_c) and np.array_equal(_np(self.k_pe), w.k_pe)
        extra = changed_pages(self.latent, self.latent_before) - set(blocks)
        assert not extra, f"untouched latent blocks written: {sorted(extra)[:8]}"
        qg = _np(self.q)
        if w.q_quant:
            assert np.array_equal(qg, w.q), "q written with Q quantisation"
            # no norm on this path: identical fp32 expressions -> bitwise codes
            assert np.array_equal(_np(self.q_out), qo), "q_out codes"
            assert np.array_equal(self.q_scale.cpu().numpy(), qs, equal_nan=True), "q_scale"
        if rc != 0:
            assert np.array_equal(qg, w.q), "q written on a flagged call"
            return {"flagged": True}
        if w.q_quant:
            rep = {"q_exact_frac": 1.0}
        else:
            # q: nope part bitwise; rope part <= 1 ulp
            assert np.array_equal(qg[..., : w.nope_dim], w.q[..., : w.nope_dim])
            d = ulp_bf16(qg[..., w.nope_dim:], q[..., w.nope_dim:])
            assert d.max() <= 1, f"q rope max ulp {d.max()}"
            rep = {"q_exact_frac": float((d == 0).mean())}
        if blocks:
            lg = _np(self.latent[idx])
            written = np.zeros(lg.shape[:2], bool)
            for b in range(w.B):
                lo, hi, L = int(self.q_indptr[b]), int(self.q_indptr[b + 1]), int(self.seq_lens[b])
                for p in range(L - (hi - lo), L):
                    written[remap[int(w.block_table[b, p // bs])], p % bs] = True
            assert np.array_equal(lg[~written], lat[~written]), "untouched latent rows"
            R = w.kv_lora_rank
            # kv_c part: same IEEE division and encoder on both sides -> bitwise
            assert np.array_equal(lg[written][:, :R], lat[written][:, :R]), "latent kv_c part"
            ulp = ulp_e4m3 if w.cache_fp8 else ulp_bf16
            d = ulp(lg[written][:, R:], lat[written][:, R:])
            assert d.max() <= 1, f"latent rope part max ulp {d.max()}"
        return rep
