"""The C ABI of libfqr.so, checked without a GPU: the library loads, exports
every function include/fqr.h declares, its parameter structs have the layout
the Python binding assumes, and host-side argument errors come back before
any CUDA call (so they can be exercised on a machine with no GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fqr.h")


@pytest.fixture(scope="module")
def fqr():
    import importlib.util
    path = os.path.join(ROOT, "qk_norm_rope_token_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_fqr_lib_build", path)
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)  # by path: the package refuses to import before the build
    build.build()
    import qk_norm_rope_token_b200 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(fqr_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    assert declared_functions() == ["fqr_append_paged", "fqr_append_plan_query",
                                    "fqr_concat_mla_cache",
                                    "fqr_pipeline_create", "fqr_pipeline_destroy",
                                    "fqr_pipeline_fork", "fqr_pipeline_join",
                                    "fqr_pipeline_submit", "fqr_pipeline_sync", "fqr_strerror"]


def test_library_exports_every_declared_symbol(fqr):
    lib = ctypes.CDLL(fqr.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", fqr.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (fqr_\w+)$", out, flags=re.M))
    assert set(declared_functions()) <= exported


@pytest.mark.parametrize("struct", ["fqr_append_params", "fqr_mla_params", "fqr_append_plan"])
def test_struct_layout_matches_binding(fqr, struct, tmp_path):
    """Compile a probe against the header and compare sizeof / offsetof of
    every field with the ctypes mirror."""
    cls = {"fqr_append_params": fqr.AppendParams, "fqr_mla_params": fqr.MlaParams,
           "fqr_append_plan": fqr.AppendPlan}[struct]
    fields = [f for f, _ in cls._fields_]
    src = tmp_path / "probe.c"
    body = "".join(f'printf("{f} %zu\\n", offsetof({struct}, {f}));\n' for f in fields)
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "fqr.h"\nint main(void){\n'
                   f'printf("sizeof %zu\\n", sizeof({struct}));\n{body}return 0;}}\n')
    exe = tmp_path / "probe"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                    str(exe)], check=True)
    got = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True,
                                                       text=True, check=True).stdout.splitlines())
    assert int(got["sizeof"]) == ctypes.sizeof(cls)
    for f in fields:
        assert int(got[f]) == getattr(cls, f).offset, f


def test_strerror(fqr):
    for code in (0, 1, 2, 3, 99):
        assert isinstance(fqr.strerror(code), str) and fqr.strerror(code)


FAKE = 1 << 20  # a 16-byte aligned non-null address; never dereferenced


def valid_append(fqr, **over):
    """A parameter set that passes every host check (never launched here)."""
    p = dict(qkv=FAKE, qkv_row_stride=10 * 128, T=4, B=4, Hq=8, Hkv=1, head_dim=128,
             q_norm_w=FAKE, k_norm_w=FAKE, eps=1e-6, cos_sin_cache=FAKE, cos_sin_rows=4096,
             rot_dim=128, rope_style=0, positions=None, q_indptr=FAKE, seq_lens=FAKE,
             page_table=FAKE, max_pages=16, k_cache=FAKE, v_cache=FAKE, num_pages=64,
             page_size=16, k_page_stride=16 * 128, v_page_stride=16 * 128, quant_policy=0,
             q_scale_inv=None, k_scale=None, v_scale=None, upper_max=448.0, out_q=FAKE,
             q_scale=None, flags=FAKE)
    p.update(over)
    return fqr.AppendParams(**p)


APPEND_BAD = {
    "head_dim_64": dict(head_dim=64),
    "hq_not_multiple": dict(Hq=6, Hkv=4, qkv_row_stride=14 * 128),
    "negative_T": dict(T=-1),
    "batch_too_large": dict(B=16385),
    "tokens_without_requests": dict(B=0),
    "page_size_zero": dict(page_size=0),
    "page_size_negative": dict(page_size=-4),
    "tail_rows_overflow": dict(B=16384, page_size=65537),
    "policy_3": dict(quant_policy=3),
    "schedule_3": dict(schedule=3),
    "schedule_negative": dict(schedule=-1),
    "rope_style_2": dict(rope_style=2),
    "rot_odd": dict(rope_style=1, rot_dim=63),
    "rot_too_big": dict(rope_style=1, rot_dim=130),
    "row_stride_short": dict(qkv_row_stride=9 * 128),
    "row_stride_unaligned": dict(qkv_row_stride=10 * 128 + 4),
    "page_stride_short": dict(k_page_stride=15 * 128),
    "null_qkv": dict(qkv=None),
    "null_out_q": dict(out_q=None),
    "null_flags": dict(flags=None),
    "null_cache": dict(v_cache=None),
    "misaligned_qkv": dict(qkv=FAKE + 8),
    "misaligned_cache": dict(k_cache=FAKE + 4),
    "misaligned_weights": dict(q_norm_w=FAKE + 2),
    "eps_nan": dict(eps=float("nan")),
    "eps_negative": dict(eps=-1.0),
    "upper_max_zero": dict(quant_policy=1, upper_max=0.0, q_scale=FAKE, k_scale=FAKE,
                           v_scale=FAKE),
    "upper_max_over_448": dict(quant_policy=1, upper_max=500.0, q_scale=FAKE, k_scale=FAKE,
                               v_scale=FAKE),
    "upper_max_inf": dict(quant_policy=1, upper_max=float("inf"), q_scale=FAKE,
                          k_scale=FAKE, v_scale=FAKE),
    "dynamic_without_q_scale": dict(quant_policy=1, k_scale=FAKE, v_scale=FAKE),
    "static_without_q_scale_inv": dict(quant_policy=2, k_scale=FAKE, v_scale=FAKE),
    "fp8_without_kv_scales": dict(quant_policy=2, q_scale_inv=FAKE),
    "fp8_page_stride_unaligned": dict(quant_policy=2, q_scale_inv=FAKE, k_scale=FAKE,
                                      v_scale=FAKE, k_page_stride=16 * 128 + 8),
    "max_seqlen_negative": dict(max_seqlen=-1),
    "norm_style_2": dict(norm_style=2),
    "out_k_without_out_v": dict(out_k=FAKE),
    "out_v_without_out_k": dict(out_v=FAKE),
    "misaligned_out_k": dict(out_k=FAKE + 8, out_v=FAKE),
    "owned_kv_null_cos_sin": dict(out_k=FAKE, out_v=FAKE, cos_sin_cache=None),
}

# caller-owned K/V rows: the paged caches, the page table and their sizes are
# not used and may be absent
OWNED_OK = dict(out_k=FAKE, out_v=FAKE, k_cache=None, v_cache=None, page_table=None,
                page_size=0, num_pages=0, max_pages=0, k_page_stride=0, v_page_stride=0)


@pytest.mark.parametrize("case", sorted(APPEND_BAD))
def test_append_host_checks_reject(fqr, case):
    assert fqr.append_paged_raw(valid_append(fqr, **APPEND_BAD[case])) == fqr.FQR_EINVAL


def test_append_neox_partial_rotary_is_unsupported(fqr):
    assert fqr.append_paged_raw(valid_append(fqr, rot_dim=64)) == fqr.FQR_ENOTSUP


def test_append_prefill_q_scale_layout_beyond_32_bit_indexing_is_unsupported(fqr):
    dyn = dict(quant_policy=1, q_scale=FAKE, k_scale=FAKE, v_scale=FAKE, B=4096, Hq=64,
               qkv_row_stride=66 * 128, Hkv=1)
    # 4096 * 64 * 8192 = 2^31 entries
    assert fqr.append_paged_raw(valid_append(fqr, max_seqlen=8192, **dyn)) == fqr.FQR_ENOTSUP


def test_append_owned_kv_needs_no_cache_or_page_table(fqr):
    """With the checks passed the call would launch, which needs a GPU: every
    host check must pass and the call must reach the CUDA runtime."""
    for over in (OWNED_OK, dict(OWNED_OK, norm_style=1),
                 dict(quant_policy=1, q_scale=FAKE, k_scale=FAKE, v_scale=FAKE, max_seqlen=129)):
        assert fqr.append_paged_raw(valid_append(fqr, **over)) == fqr.FQR_ECUDA


def test_plan_query_checks_like_the_call(fqr):
    """fqr_append_plan_query applies fqr_append_paged's host checks, returns
    their codes, and answers an empty batch without touching the device."""
    plan = fqr.AppendPlan()
    assert fqr.LIB.fqr_append_plan_query(ctypes.byref(valid_append(fqr)), None) == fqr.FQR_EINVAL
    for case in sorted(APPEND_BAD):
        rc = fqr.LIB.fqr_append_plan_query(ctypes.byref(valid_append(fqr, **APPEND_BAD[case])),
                                           ctypes.byref(plan))
        assert rc == fqr.FQR_EINVAL, case
    assert fqr.LIB.fqr_append_plan_query(ctypes.byref(valid_append(fqr, rot_dim=64)),
                                         ctypes.byref(plan)) == fqr.FQR_ENOTSUP
    p = valid_append(fqr, T=0, B=0, qkv=None, out_q=None, q_indptr=None, seq_lens=None,
                     page_table=None, flags=None)
    plan.grid = 7
    assert fqr.LIB.fqr_append_plan_query(ctypes.byref(p), ctypes.byref(plan)) == fqr.FQR_OK
    assert (plan.schedule, plan.grid, plan.block_threads, plan.tasks) == (0, 0, 0, 0)
    # valid parameters need the device's occupancy: on a machine without a GPU
    # the query reaches the CUDA runtime and reports that
    assert fqr.LIB.fqr_append_plan_query(ctypes.byref(valid_append(fqr)),
                                         ctypes.byref(plan)) == fqr.FQR_ECUDA


def test_append_null_params(fqr):
    assert fqr.LIB.fqr_append_paged(None, None) == fqr.FQR_EINVAL
    assert fqr.LIB.fqr_concat_mla_cache(None, None) == fqr.FQR_EINVAL


def test_empty_batch_returns_ok_without_launching(fqr):
    # T == 0 and B == 0: nothing to do, no CUDA call (this machine has no GPU)
    p = valid_append(fqr, T=0, B=0, qkv=None, out_q=None, q_indptr=None, seq_lens=None,
                     page_table=None, flags=None)
    assert fqr.append_paged_raw(p) == fqr.FQR_OK
    m = fqr.MlaParams(T=0, B=0)
    assert fqr.concat_mla_cache_raw(m) == fqr.FQR_OK


def valid_mla(fqr, **over):
    p = dict(q=FAKE, T=32, B=32, Hq=128, nope_dim=128, rope_dim=64, q_token_stride=128 * 192,
             q_head_stride=192, kv_c=FAKE, kv_lora_rank=512, kv_c_stride=512, k_pe=FAKE,
             k_pe_stride=64, cos_sin_cache=FAKE, cos_sin_rows=32768, rope_style=1,
             positions=None, q_indptr=FAKE, seq_lens=FAKE, block_table=FAKE, max_blocks=512,
             latent_cache=FAKE, num_blocks=16384, block_size=64, cache_fp8=1, kv_scale=FAKE,
             flags=FAKE)
    p.update(over)
    return fqr.MlaParams(**p)


MLA_BAD = {
    "block_size_zero": (dict(block_size=0), 1),
    "cache_fp8_without_scale": (dict(kv_scale=None), 1),
    "null_latent": (dict(latent_cache=None), 1),
    "misaligned_latent": (dict(latent_cache=FAKE + 8), 1),
    "head_stride_short": (dict(q_head_stride=128), 1),
    "rope_dim_odd": (dict(rope_dim=63), 1),
    "rope_dim_32": (dict(rope_dim=32, q_head_stride=160, q_token_stride=128 * 160,
                         k_pe_stride=32), 2),
    "rank_not_multiple_of_8": (dict(kv_lora_rank=500, kv_c_stride=500), 2),
    "q_quant_5": (dict(q_quant=5, q_out=FAKE, q_scale=FAKE), 1),
    "q_group_zero": (dict(q_quant=4, q_out=FAKE, q_scale=FAKE, q_group=0), 1),
    "q_group_not_multiple_of_8": (dict(q_quant=4, q_out=FAKE, q_scale=FAKE, q_group=60), 1),
    "q_group_without_q_scale": (dict(q_quant=4, q_out=FAKE, q_group=64), 1),
    "q_static_without_scale": (dict(q_quant=1, q_out=FAKE), 1),
    "q_dynamic_without_q_scale": (dict(q_quant=2, q_out=FAKE), 1),
    "q_dynamic_upper_max_zero": (dict(q_quant=3, q_out=FAKE, q_scale=FAKE, upper_max=0.0), 1),
    "q_quant_without_q_out": (dict(q_quant=2, q_scale=FAKE), 1),
    "q_out_misaligned": (dict(q_quant=1, q_scale_inv=FAKE, q_out=FAKE + 8), 1),
    "q_quant_nope_not_multiple_of_8": (dict(q_quant=1, q_scale_inv=FAKE, q_out=FAKE,
                                            nope_dim=124, q_head_stride=188,
                                            q_token_stride=128 * 188), 2),
}


@pytest.mark.parametrize("case", sorted(MLA_BAD))
def test_mla_host_checks_reject(fqr, case):
    over, code = MLA_BAD[case]
    assert fqr.concat_mla_cache_raw(valid_mla(fqr, **over)) == code


def test_pipeline_rejects_bad_arguments_before_any_cuda_call(fqr):
    import ctypes
    h = ctypes.c_void_p()
    good = (fqr.AppendParams * 1)(valid_append(fqr))
    ptrs = (ctypes.c_void_p * 1)(FAKE)
    L = fqr.LIB
    assert L.fqr_pipeline_create(0, good, ptrs, 256, ptrs, 256, ctypes.byref(h)) == fqr.FQR_EINVAL
    assert L.fqr_pipeline_create(9, good, ptrs, 256, ptrs, 256, ctypes.byref(h)) == fqr.FQR_EINVAL
    assert L.fqr_pipeline_create(1, None, ptrs, 256, ptrs, 256, ctypes.byref(h)) == fqr.FQR_EINVAL
    assert L.fqr_pipeline_create(1, good, ptrs, 0, ptrs, 256, ctypes.byref(h)) == fqr.FQR_EINVAL
    nul = (ctypes.c_void_p * 1)(None)
    assert L.fqr_pipeline_create(1, good, nul, 256, ptrs, 256, ctypes.byref(h)) == fqr.FQR_EINVAL
    bad = (fqr.AppendParams * 1)(valid_append(fqr, head_dim=64))
    assert L.fqr_pipeline_create(1, bad, ptrs, 256, ptrs, 256, ctypes.byref(h)) == fqr.FQR_EINVAL
    empty = (fqr.AppendParams * 1)(valid_append(fqr, T=0, B=0))
    assert L.fqr_pipeline_create(1, empty, ptrs, 256, ptrs, 256, ctypes.byref(h)) == fqr.FQR_EINVAL
    assert not h.value
    for name in ("fqr_pipeline_sync", "fqr_pipeline_destroy"):
        assert getattr(L, name)(None) == fqr.FQR_EINVAL
    assert L.fqr_pipeline_submit(None, FAKE, FAKE) == fqr.FQR_EINVAL
    assert L.fqr_pipeline_join(None, None) == fqr.FQR_EINVAL
    assert L.fqr_pipeline_fork(None, None) == fqr.FQR_EINVAL


def test_floor_copy_library_loads_and_checks_arguments():
    """libfqr_floor.so (the bench's plain copy kernel) exports fqr_floor_copy
    and rejects invalid arguments before any CUDA call."""
    import ctypes
    path = os.path.join(ROOT, "qk_norm_rope_token_b200", "libfqr_floor.so")
    lib = ctypes.CDLL(path)
    f = lib.fqr_floor_copy
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64,
                  ctypes.c_int, ctypes.c_void_p]
    f.restype = ctypes.c_int
    assert f(FAKE, FAKE, 24, 32, 4, None) == 1          # size not a multiple of 16
    assert f(FAKE + 8, FAKE, 32, 32, 4, None) == 1      # misaligned source
    assert f(None, FAKE, 32, 32, 4, None) == 1          # no source
    assert f(FAKE, FAKE, 32, 32, 0, None) == 1          # no blocks
