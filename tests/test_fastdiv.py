"""Host check of the kernels' division by run-time invariant integers
(multiply-high and shift): exact for every dividend in [0, 2^31)."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_fastdiv_exact(tmp_path):
    exe = tmp_path / "fastdiv_check"
    subprocess.run(["nvcc", "-x", "cu", "-O2", "-std=c++17",
                    "-gencode", "arch=compute_100a,code=sm_100a", "-I",
                    os.path.join(ROOT, "qk_norm_rope_token_b200", "csrc"),
                    os.path.join(ROOT, "tests", "csrc", "fastdiv_check.cpp"), "-o", str(exe)],
                   check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout
    assert "bad=0" in r.stdout
