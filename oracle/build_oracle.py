"""Compile the CPU oracle (``attention_oracle.c``, ``fp8_oracle.c``) into
``liboracle.so``.

Test infrastructure: building the checker is not using it.  Plain gcc, -O2,
OpenMP, no -ffast-math (the oracle relies on IEEE exp/log and ordered sums).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRCS = [os.path.join(HERE, "attention_oracle.c"),
        os.path.join(HERE, "fp8_oracle.c")]
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(s) for s in SRCS)):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-fno-fast-math",
           "-fopenmp", "-fPIC", "-shared"] + SRCS + ["-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
