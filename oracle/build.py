"""Build the C oracle in-tree (oracle/_lib/libmoe_oracle.so). Test infrastructure only."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "_lib")
SRC = os.path.join(HERE, "moe_oracle.c")
OUT = os.path.join(LIB, "libmoe_oracle.so")

# -ffp-contract=off keeps every a*b+c as two roundings unless the source says fmaf;
# no -ffast-math: IEEE division, rounding and subnormals as written.
CFLAGS = ["-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
          "-std=gnu11", "-Wall", "-Wno-unused-result"]


def build(force: bool = False) -> str:
    os.makedirs(LIB, exist_ok=True)
    if force or not os.path.exists(OUT) or os.path.getmtime(SRC) > os.path.getmtime(OUT):
        subprocess.check_call(["gcc", *CFLAGS, "-o", OUT, SRC, "-lm"])
    return OUT


if __name__ == "__main__":
    print(build(force=True))
