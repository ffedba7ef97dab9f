"""Builds gen/libmoe_gen.so with gcc (OpenMP)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_gen.c")
OUT = os.path.join(HERE, "libmoe_gen.so")


def build(force: bool = False) -> str:
    if force or not os.path.exists(OUT) or os.path.getmtime(OUT) < os.path.getmtime(SRC):
        tmp = OUT + ".tmp.%d" % os.getpid()
        tmpdir = os.path.join(HERE, "_build", "tmp")   # the compiler's temporaries stay in the repository
        os.makedirs(tmpdir, exist_ok=True)
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                               SRC, "-o", tmp, "-lm"], env=dict(os.environ, TMPDIR=tmpdir))
        os.replace(tmp, OUT)
    return OUT


def ensure_built() -> str:
    return build(False)


if __name__ == "__main__":
    print(build(True))
