"""Builds oracle/libmoe_oracle.so with gcc.

No -ffast-math and -ffp-contract=off: the oracle's fp32 router order and its
fp64 sums must be exactly the ones written in the source.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_oracle.c")
OUT = os.path.join(HERE, "libmoe_oracle.so")


def build(force: bool = False, out: str = OUT, defines=()) -> str:
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(SRC):
        tmp = out + ".tmp.%d" % os.getpid()
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]
        cmd += ["-D%s" % d for d in defines]
        subprocess.check_call(cmd + [SRC, "-o", tmp, "-lm"])
        os.replace(tmp, out)
    return out


def ensure_built() -> str:
    return build(False)


if __name__ == "__main__":
    print(build(True))
