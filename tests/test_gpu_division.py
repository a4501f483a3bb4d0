"""GPU checks of the payload divisions (one Markstein correction on a correctly
rounded reciprocal) against IEEE division.  Dynamic Q: bit-equal quotients for
a = +-0 or |a| >= 2^-100 with a normal quotient, and equal E4M3 codes
wherever |a / b| <= 448, over
every binary32 dividend for divisors across the q_scale range and over 2^33
random pairs.  K / V (guarded, any value and scale): equal E4M3 codes over
every binary32 dividend for a set of scales, inside and outside the guard, and
over 2^32 random lanes of 16 mixed values."""
import os
import subprocess

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    exe = tmp_path_factory.mktemp("div") / "division_check"
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-I", os.path.join(ROOT, "qk_norm_rope_token_b200", "csrc"),
                    os.path.join(ROOT, "tests", "csrc", "division_check.cu"), "-o", str(exe)],
                   check=True)
    return str(exe)


# q_scale = max(amax, 1e-6) / 448 for amax = 1e-6 (the floor), 1, 3.7, 10 and
# 1000; plus 1.0, a significand of all ones, and a large scale
DIVISORS = ["31196446", "3b124925", "3c075075", "3cb6db6e", "400edb6e", "3f800000",
            "3f7fffff", "4e6b79a3"]


@pytest.mark.parametrize("bits", DIVISORS)
def test_every_dividend(checker, bits):
    r = subprocess.run([checker, "all", bits], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr


@pytest.mark.parametrize("seed", [1, 2])
def test_random_pairs(checker, seed):
    r = subprocess.run([checker, "rand", str(seed), str(1 << 32)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr


# K / V scales: 0.05 and 0.02 (the workloads' scales), 1, a significand of all
# ones, the guard's ends 2^-80 and 2^80, and 1e-30, 1e30 and -0.05 (outside
# it: IEEE division)
KV_SCALES = ["3d4ccccd", "3ca3d70a", "3f800000", "3f7fffff", "17800000", "67800000",
             "0da24260", "7149f2ca", "bd4ccccd"]


@pytest.mark.parametrize("bits", KV_SCALES)
def test_kv_every_dividend(checker, bits):
    r = subprocess.run([checker, "kvall", bits], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr


def test_kv_random_lanes(checker):
    r = subprocess.run([checker, "kvrand", "3", str(1 << 32)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
