"""Build the oracle's shared library (test infrastructure only).

Compiles bitnet_oracle.c single-threaded with -O2 -ffp-contract=off so that every
fp32 expression in it rounds exactly as written (no fused multiply-add).
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "bitnet_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")
CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-shared", "-fPIC", "-Wall"]


def build(force: bool = False, src: str = SRC, out: str = LIB, extra=()) -> str:
    """Compile ``src`` into ``out`` unless ``out`` is newer than ``src``."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    cmd = ["gcc", *CFLAGS, *extra, "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(force=True))
