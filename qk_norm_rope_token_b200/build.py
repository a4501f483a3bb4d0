"""Build libfqr.so (the CUDA library behind include/fqr.h) for sm_100a.

    python qk_norm_rope_token_b200/build.py [--force] [--verbose-ptxas]

nvcc cross-compiles on a machine without a GPU.  The library is built in-tree
(qk_norm_rope_token_b200/libfqr.so) with the CUDA runtime linked statically.
No fast-math: divisions and square roots stay IEEE-rounded.
"""
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libfqr.so")
SOURCES = ["fqr_api.cu", "fqr_append.cu", "fqr_append_warp.cu", "fqr_append_pipe.cu",
           "fqr_mla.cu", "fqr_runtime.cu"]
DEPS = ["fqr_device.cuh", "fqr_head.cuh", "fqr_launch.h"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
    "-DNDEBUG",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    inputs = [os.path.join(CSRC, f) for f in SOURCES + DEPS] + [os.path.join(INCLUDE, "fqr.h")]
    return os.path.getmtime(LIB) < max(os.path.getmtime(f) for f in inputs)


FLOOR_SRC = os.path.join(CSRC, "copy_floor.cu")
FLOOR_LIB = os.path.join(PKG, "libfqr_floor.so")


def build_floor(force: bool = False) -> str:
    """libfqr_floor.so: the bench's plain copy kernel (not part of libfqr)."""
    if (not force and os.path.exists(FLOOR_LIB)
            and os.path.getmtime(FLOOR_LIB) >= os.path.getmtime(FLOOR_SRC)):
        return FLOOR_LIB
    tmp = FLOOR_LIB + ".tmp%d" % os.getpid()
    subprocess.run([nvcc(), *NVCC_FLAGS, "-shared", FLOOR_SRC, "-o", tmp], check=True)
    os.replace(tmp, FLOOR_LIB)
    return FLOOR_LIB


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    build_floor(force)
    if not force and not _stale():
        return LIB
    flags = list(NVCC_FLAGS)
    if verbose_ptxas:
        flags += ["-Xptxas", "-v"]
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = [nvcc(), *flags, "-shared", "-I", INCLUDE, "-I", CSRC,
           *[os.path.join(CSRC, f) for f in SOURCES], "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--verbose-ptxas" in sys.argv))
