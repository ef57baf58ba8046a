"""Build the C oracle (``nf4_oracle.c``) into ``liboracle_nf4.so`` beside it.

Test infrastructure: compiled by the package build step so that the checker
exists wherever the tests run; the product library never loads it.
Flags: -O2 -ffp-contract=off (no FMA contraction), no fast-math.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "nf4_oracle.c")
LIB = os.path.join(HERE, "liboracle_nf4.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
           "-fPIC", "-shared", "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
