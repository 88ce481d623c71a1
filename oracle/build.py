"""Compile the C oracle into oracle/liborc.so (test infrastructure only).

The flags keep binary32 arithmetic exact IEEE: no fast-math and no FMA
contraction, so every `float` operation in orc.c rounds once, to nearest even.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "orc.c")
LIB = os.path.join(HERE, "liborc.so")

CFLAGS = ["-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
          "-Wall", "-Wextra", "-Werror"]


def build_oracle(src: str = SRC, out: str = LIB, extra_flags=(), force: bool = False) -> str:
    """Build `src` into the shared library `out` (skipped when up to date)."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)
            and not extra_flags):
        return out
    cmd = ["gcc", *CFLAGS, *extra_flags, "-shared", "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build_oracle(force=True))
