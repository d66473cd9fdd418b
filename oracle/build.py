"""Compile the fp64 C oracle into ``oracle/liblaoracle.so``.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  Plain gcc, IEEE fp64:
no fast-math and no FMA contraction, so every sum is evaluated in the loop
order the C source spells out.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "la_oracle.c")
LIB = os.path.join(HERE, "liblaoracle.so")


def build(force: bool = False, out: str = LIB, defines=()) -> str:
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(SRC):
        return out
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC", "-pthread",
           *[f"-D{d}" for d in defines], SRC, "-o", out + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
