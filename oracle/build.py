"""Build the CPU oracle (plain C, gcc) into oracle/liboracle_moe.so.

The oracle is test infrastructure: this build step exists so the tests, the
smoke check and the benchmark's CPU-baseline leg can load it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle_moe.c")
LIB = os.path.join(HERE, "liboracle_moe.so")


def build(force: bool = False) -> str:
    deps = [SRC, os.path.join(HERE, "oracle_moe.h")]
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(p) for p in deps)):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-Wall", "-Wextra",
           "-o", tmp, SRC, "-lm", "-lpthread"]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
