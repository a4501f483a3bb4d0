"""Exhaustive GPU sweeps over all 2^32 binary32 inputs, and a bounded wait
that runs out on purpose.

- The kernels' packed encoders (fqr::pack_e4m3x2, fqr::pack_bf16x2) against
  the oracle's E4M3 and BF16 encoders, which are themselves pinned against a
  brute-force nearest-value search over all 2^32 inputs on the CPU
  (tests/test_oracle_encoders.py): RN satfinite E4M3 and RNE BF16, as the
  FlashInfer PR #5956 "Contract" states them, for every value the kernels may
  pack, not only BF16-valued ones.
- The inverse RMS's 1 / sqrt(v) (fqr::rn_recip_sqrt) against CUDA's correctly
  rounded __frcp_rn(__fsqrt_rn(v)): the definition's two roundings.

- The library's bounded wait (tests/csrc/wait_timeout_check.cu): with a
  50 ms budget, a wait on an mbarrier that nothing arrives at gives up, the
  kernel returns, every flag reads -2 and the context stays usable.

Each check is a small CUDA program under tests/csrc, built here with nvcc
(the pack sweep links the oracle's C source)."""
import os
import subprocess

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NVCC = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
        "-I", os.path.join(ROOT, "qk_norm_rope_token_b200", "csrc")]


def _build(tmp_path_factory, name, extra=()):
    exe = tmp_path_factory.mktemp(name) / name
    subprocess.run(NVCC + list(extra) + [os.path.join(ROOT, "tests", "csrc", name + ".cu"),
                                         "-o", str(exe)], check=True)
    return str(exe)


def test_packs_match_the_oracle_encoders_on_every_input(tmp_path_factory):
    exe = _build(tmp_path_factory, "pack_check",
                 ["-I", os.path.join(ROOT, "oracle"), "-Xcompiler", "-ffp-contract=off",
                  os.path.join(ROOT, "oracle", "fqr_oracle.c")])
    r = subprocess.run([exe], capture_output=True, text=True)
    print(r.stdout)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "pack_e4m3x2: 0 mismatches" in r.stdout and "pack_bf16x2: 0 mismatches" in r.stdout


def test_recip_sqrt_matches_the_correctly_rounded_steps_on_every_input(tmp_path_factory):
    exe = _build(tmp_path_factory, "recip_sqrt_check")
    r = subprocess.run([exe], capture_output=True, text=True)
    print(r.stdout)
    assert r.returncode == 0, r.stdout + r.stderr


def test_a_wait_that_runs_out_returns_and_reports(tmp_path_factory):
    """The library's bounded wait, with a 50 ms budget in a test build, on an
    mbarrier nothing arrives at: the kernel returns and every flag reads the
    timeout code -2 (atomicMin over a valid call's 0), and the context stays
    usable."""
    exe = _build(tmp_path_factory, "wait_timeout_check")
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    print(r.stdout)
    assert r.returncode == 0, r.stdout + r.stderr
