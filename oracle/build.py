"""Builds oracle/libmoe_oracle.so with gcc.

No -ffast-math and -ffp-contract=off: the oracle's fp32 router order and its
fp64 sums must be exactly the ones written in the source.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_oracle.c")
OUT = os.path.join(HERE, "libmoe_oracle.so")
GDN_SRC = os.path.join(HERE, "gdn_oracle.c")
GDN_OUT = os.path.join(HERE, "libgdn_oracle.so")


def _env() -> dict:
    """The compiler's temporary files go to a folder inside the repository."""
    tmpdir = os.path.join(HERE, "_build", "tmp")
    os.makedirs(tmpdir, exist_ok=True)
    return dict(os.environ, TMPDIR=tmpdir)


def build(force: bool = False, out: str = OUT, defines=(), src: str = SRC) -> str:
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + ".tmp.%d" % os.getpid()
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]
        cmd += ["-D%s" % d for d in defines]
        subprocess.check_call(cmd + [src, "-o", tmp, "-lm"], env=_env())
        os.replace(tmp, out)
    return out


def ensure_built() -> str:
    return build(False)


def build_gdn(force: bool = False, out: str = GDN_OUT, src: str = GDN_SRC) -> str:
    """The recurrent-scan oracle (a separate library, same compiler flags)."""
    return build(force, out=out, src=src)


def ensure_gdn_built() -> str:
    return build_gdn(False)


if __name__ == "__main__":
    print(build(True))
    print(build_gdn(True))
