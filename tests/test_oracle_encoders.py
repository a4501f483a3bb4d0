"""Pins of the oracle's BF16 and FP8 E4M3 encoders against the format
definitions: exhaustive brute force over all 2^32 binary32 inputs, round trips
over every code, and hand-worked golden points."""
import os
import subprocess

import numpy as np
import pytest

import oracle
from tests._util import e4m3_brute, e4m3_value_table, read_golden

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def brute_bin(tmp_path_factory):
    out = tmp_path_factory.mktemp("brute") / "brute_encoders"
    subprocess.run(
        ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-I", os.path.join(ROOT, "oracle"),
         os.path.join(ROOT, "tests", "csrc", "brute_encoders.c"),
         os.path.join(ROOT, "oracle", "fqr_oracle.c"), "-o", str(out), "-lm", "-lpthread"],
        check=True)
    return str(out)


@pytest.mark.parametrize("fmt", ["e4m3", "bf16"])
def test_exhaustive_bruteforce(brute_bin, fmt):
    """Every binary32 bit pattern encodes to the nearest value found by
    brute-force search (ties to even; E4M3 saturating at +-448)."""
    threads = str(max(1, os.cpu_count() or 1))
    r = subprocess.run([brute_bin, fmt, threads], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "mismatches=0 " in r.stdout


def test_e4m3_every_code_round_trips():
    vals = e4m3_value_table()
    for c in range(256):
        v = np.float32(vals[c])
        got = int(oracle.e4m3(np.array([v]))[0])
        if np.isnan(vals[c]):
            assert got == 0x7F
        else:
            assert got == c, (hex(c), float(v), hex(got))


def test_bf16_every_code_round_trips():
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = (codes.astype(np.uint32) << 16).view(np.float32)
    got = oracle.bf16(vals)
    nan = np.isnan(vals)
    assert np.array_equal(got[~nan], codes[~nan])
    assert np.all(np.isnan((got[nan].astype(np.uint32) << 16).view(np.float32)))


@pytest.mark.parametrize("name,fn", [("e4m3_points.txt", oracle.e4m3),
                                     ("bf16_points.txt", oracle.bf16)])
def test_golden_points(name, fn):
    for bits, want, note in read_golden(name):
        x = np.array([bits], dtype=np.uint32).view(np.float32)
        got = int(fn(x)[0])
        assert got == want, (note, hex(bits), hex(got), hex(want))


def test_e4m3_matches_numpy_bruteforce_random():
    """A second, vectorised brute force (numpy table search) on 2^20 random
    bit patterns concentrated on the E4M3 range."""
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(1 << 20) * np.exp2(rng.uniform(-12, 10, 1 << 20))).astype(np.float32)
    assert np.array_equal(oracle.e4m3(x), e4m3_brute(x))
