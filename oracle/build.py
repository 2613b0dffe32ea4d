"""Build the CPU oracle (plain C) into oracle/libzipnn_oracle.so.

Test infrastructure: the library built here is loaded only by the tests, the smoke
check and the benchmark's CPU baseline.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "zipnn_oracle.c")
LIB = os.path.join(HERE, "libzipnn_oracle.so")

# -ffp-contract=off: every double operation of the grouping step rounds on its own,
# so a device implementation without fused multiply-add can match it bit for bit.
CFLAGS = ["-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-Wall", "-Wextra", "-D_POSIX_C_SOURCE=200809L"]


def build(force=False):
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= max(
            os.path.getmtime(SRC), os.path.getmtime(os.path.join(HERE, "zipnn_oracle.h"))):
        return LIB
    cmd = ["gcc", *CFLAGS, SRC, "-o", LIB + ".tmp", "-lpthread"]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
