"""GPU test of the pipelined host-memory API (StagedAppend over the native
fqr_pipeline_*): the host results and the final caches of batches submitted
through it match the CPU oracle run on the same batches in the same order
(flags and V bitwise, out_q and K within 1 ulp, q_scale within 1e-5 relative),
for every pipeline depth, and a stream joined after the submits sees them
done."""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import qk_norm_rope_token_b200 as fqr
    from tests.gpu_harness import _dev, _np, fill_random_
    from tests._util import ulp_bf16, ulp_e4m3

DEV = "cuda"


def _batches(n, policy):
    """n decode batches of 16 requests on one cache; they share the first
    batch's norm weights (a pipeline holds one set of weights)."""
    ws = []
    for i in range(n):
        rng = np.random.default_rng(100 + i)
        L = rng.integers(1, 200, 16)
        w = workloads.make_append(seed=200 + i, n_new=[1] * 16, seq_lens=L, Hq=8, Hkv=2,
                                  page_size=16, max_pages=13, num_pages=300,
                                  quant_policy=policy, q_scale_inv=20.0, k_scale=0.05,
                                  v_scale=0.05, cos_sin_rows=256)
        if ws:
            w.q_norm_w, w.k_norm_w = ws[0].q_norm_w, ws[0].k_norm_w
        ws.append(w)
    return ws


@pytest.mark.parametrize("depth", [1, 2, 3])
@pytest.mark.parametrize("policy", [0, 1])
def test_staged_matches_oracle(depth, policy):
    ws = _batches(7, policy)
    w0 = ws[0]
    es = w0.kv_esize
    dt = torch.int16 if es == 2 else torch.uint8
    shape = (w0.num_pages, w0.page_size, w0.Hkv, 128)
    kc = torch.empty(shape, dtype=dt, device=DEV)
    vc = torch.empty(shape, dtype=dt, device=DEV)
    fill_random_(kc, 1)
    fill_random_(vc, 2)
    # the oracle: the same batches, in the same order, on host copies of the
    # initial caches (batches may share pages, so the order matters)
    ok, ov = _np(kc).copy(), _np(vc).copy()
    want = []
    for w in ws:
        oq, qs, fl = oracle.new_outputs(w)
        assert oracle.append_paged(w, ok, ov, oq, qs if policy == 1 else None, fl) == 0
        want.append((oq, fl, qs))
    cs, qw, kw_ = _dev(w0.cos_sin), _dev(w0.q_norm_w), _dev(w0.k_norm_w)
    scales = {k: torch.tensor([getattr(w0, k)], dtype=torch.float32, device=DEV)
              for k in ("q_scale_inv", "k_scale", "v_scale")}
    qdt = dt if policy == 0 else torch.uint8
    kw = dict(q_norm_w=qw, k_norm_w=kw_, eps=w0.eps, quant_policy=policy,
              k_scale=scales["k_scale"] if policy else None,
              v_scale=scales["v_scale"] if policy else None, upper_max=w0.upper_max)
    in_shapes = {"qkv": ((w0.T, w0.row_stride), torch.int16), "q_indptr": ((w0.B + 1,), torch.int32),
                 "seq_lens": ((w0.B,), torch.int32),
                 "page_table": (tuple(w0.page_table.shape), torch.int32)}
    out_shapes = {"out_q": ((w0.T, w0.Hq, 128), qdt), "flags": ((w0.B,), torch.int32)}
    if policy == 1:
        out_shapes["q_scale"] = ((w0.T, w0.Hq), torch.float32)
    sa = fqr.StagedAppend(in_shapes, out_shapes, DEV, depth=depth, cos_sin_cache=cs,
                          k_cache=kc, v_cache=vc, **kw)
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
    ulp = ulp_bf16 if policy == 0 else ulp_e4m3
    for (oq, fl, qs), ho in zip(want, host_out):
        assert np.array_equal(ho["flags"].numpy(), fl)
        got_q = ho["out_q"].numpy()
        got_q = got_q.view(np.uint16) if got_q.dtype == np.int16 else got_q
        assert ulp(got_q, oq).max() <= 1
        if policy == 1:
            g = ho["q_scale"].numpy()
            assert (np.abs(g - qs) / np.abs(qs)).max() <= 1e-5
    assert np.array_equal(_np(vc), ov), "V cache"
    assert ulp(_np(kc), ok).max() <= 1, "K cache"


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
