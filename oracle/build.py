"""Build the CPU oracle (oracle/liboracle.so) with gcc.

Test infrastructure: the oracle is compiled without FMA contraction and without
fast-math so that every fp32 product and sum is rounded on its own, exactly as
the oracle's source states it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fqr_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = ["-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
          "-Wall", "-Wextra", "-Werror"]


def build(force: bool = False) -> str:
    """Compile liboracle.so if it is missing or older than its sources."""
    srcs = [SRC, os.path.join(HERE, "fqr_oracle.h")]
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(s) for s in srcs)):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", *CFLAGS, "-shared", SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
