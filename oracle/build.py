"""Build the CPU oracle shared library (test infrastructure only).

Compiles ``bnb4_oracle.c`` with plain gcc: ``-O2 -ffp-contract=off
-fno-fast-math`` so every fp32 operation is a separately rounded IEEE
operation (x86-64 SSE, no x87, no fused multiply-add contraction).
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "bnb4_oracle.c")
LIB = os.path.join(HERE, "liborc_bnb4.so")

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
          "-fPIC", "-shared", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile the oracle if the library is missing or older than its source."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
