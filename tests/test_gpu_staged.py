"""GPU test of the pipelined host-memory API (StagedAppend over the native
fqr_pipeline_*): the same batches submitted through it give bitwise the same
host results and the same caches as sequential append_paged calls, for every
pipeline depth, and a stream joined after the submits sees them done."""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import qk_norm_rope_token_b200 as fqr
    from tests.gpu_harness import _dev, fill_random_

DEV = "cuda"


def _batches(n, policy):
    ws = []
    for i in range(n):
        rng = np.random.default_rng(100 + i)
        L = rng.integers(1, 200, 16)
        ws.append(workloads.make_append(seed=200 + i, n_new=[1] * 16, seq_lens=L, Hq=8, Hkv=2,
                                        page_size=16, max_pages=13, num_pages=300,
                                        quant_policy=policy, q_scale_inv=20.0, k_scale=0.05,
                                        v_scale=0.05, cos_sin_rows=256))
    return ws


@pytest.mark.parametrize("depth", [1, 2, 3])
@pytest.mark.parametrize("policy", [0, 1])
def test_staged_matches_sequential(depth, policy):
    ws = _batches(7, policy)
    w0 = ws[0]
    es = w0.kv_esize
    dt = torch.int16 if es == 2 else torch.uint8
    shape = (w0.num_pages, w0.page_size, w0.Hkv, 128)
    caches = {}
    for name in ("seq", "staged"):
        k = torch.empty(shape, dtype=dt, device=DEV)
        v = torch.empty(shape, dtype=dt, device=DEV)
        fill_random_(k, 1)
        fill_random_(v, 2)
        caches[name] = (k, v)
    cs, qw, kw_ = _dev(w0.cos_sin), _dev(w0.q_norm_w), _dev(w0.k_norm_w)
    scales = {k: torch.tensor([getattr(w0, k)], dtype=torch.float32, device=DEV)
              for k in ("q_scale_inv", "k_scale", "v_scale")}
    qdt = dt if policy == 0 else torch.uint8
    kw = dict(q_norm_w=qw, k_norm_w=kw_, eps=w0.eps, quant_policy=policy,
              k_scale=scales["k_scale"] if policy else None,
              v_scale=scales["v_scale"] if policy else None, upper_max=w0.upper_max)
    # sequential reference
    seq_out = []
    for w in ws:
        out_q = torch.empty((w.T, w.Hq, 128), dtype=qdt, device=DEV)
        flags = torch.empty((w.B,), dtype=torch.int32, device=DEV)
        q_scale = torch.empty((w.T, w.Hq), dtype=torch.float32, device=DEV) if policy == 1 else None
        fqr.append_paged(_dev(w.qkv), cs, _dev(w.q_indptr), _dev(w.seq_lens), _dev(w.page_table),
                         *caches["seq"], out_q, flags, q_scale=q_scale, **kw)
        seq_out.append((out_q.cpu(), flags.cpu(), None if q_scale is None else q_scale.cpu()))
    # pipelined
    in_shapes = {"qkv": ((w0.T, w0.row_stride), torch.int16), "q_indptr": ((w0.B + 1,), torch.int32),
                 "seq_lens": ((w0.B,), torch.int32),
                 "page_table": (tuple(w0.page_table.shape), torch.int32)}
    out_shapes = {"out_q": ((w0.T, w0.Hq, 128), qdt), "flags": ((w0.B,), torch.int32)}
    if policy == 1:
        out_shapes["q_scale"] = ((w0.T, w0.Hq), torch.float32)
    sa = fqr.StagedAppend(in_shapes, out_shapes, DEV, depth=depth, cos_sin_cache=cs,
                          k_cache=caches["staged"][0], v_cache=caches["staged"][1], **kw)
    host_out = []
    for w in ws:
        hi, ho = sa.new_host_buffers()
        hi["qkv"].copy_(torch.from_numpy(w.qkv.view(np.int16)))
        hi["q_indptr"].copy_(torch.from_numpy(w.q_indptr))
        hi["seq_lens"].copy_(torch.from_numpy(w.seq_lens))
        hi["page_table"].copy_(torch.from_numpy(w.page_table))
        sa.submit(hi, ho)
        host_out.append(ho)
    sa.synchronize()
    sa.close()
    for (oq, fl, qs), ho in zip(seq_out, host_out):
        assert torch.equal(oq, ho["out_q"]) and torch.equal(fl, ho["flags"])
        if qs is not None:
            assert torch.equal(qs, ho["q_scale"])
    assert torch.equal(caches["seq"][0], caches["staged"][0])
    assert torch.equal(caches["seq"][1], caches["staged"][1])


def test_join_orders_a_stream_after_the_batches():
    ws = _batches(4, 0)
    w0 = ws[0]
    shape = (w0.num_pages, w0.page_size, w0.Hkv, 128)
    kc = torch.zeros(shape, dtype=torch.int16, device=DEV)
    vc = torch.zeros(shape, dtype=torch.int16, device=DEV)
    in_shapes = {"qkv": ((w0.T, w0.row_stride), torch.int16), "q_indptr": ((w0.B + 1,), torch.int32),
                 "seq_lens": ((w0.B,), torch.int32),
                 "page_table": (tuple(w0.page_table.shape), torch.int32)}
    out_shapes = {"out_q": ((w0.T, w0.Hq, 128), torch.int16), "flags": ((w0.B,), torch.int32)}
    sa = fqr.StagedAppend(in_shapes, out_shapes, DEV, depth=2, cos_sin_cache=_dev(w0.cos_sin),
                          k_cache=kc, v_cache=vc, q_norm_w=_dev(w0.q_norm_w),
                          k_norm_w=_dev(w0.k_norm_w))
    hos = []
    for w in ws:
        hi, ho = sa.new_host_buffers()
        hi["qkv"].copy_(torch.from_numpy(w.qkv.view(np.int16)))
        hi["q_indptr"].copy_(torch.from_numpy(w.q_indptr))
        hi["seq_lens"].copy_(torch.from_numpy(w.seq_lens))
        hi["page_table"].copy_(torch.from_numpy(w.page_table))
        ho["flags"].fill_(77)
        sa.submit(hi, ho)
        hos.append(ho)
    s = torch.cuda.Stream()
    sa.join(s)
    ev = torch.cuda.Event()
    ev.record(s)
    ev.synchronize()
    assert all(int(ho["flags"].abs().max()) == 0 for ho in hos)
    sa.close()
