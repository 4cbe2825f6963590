"""Compiles the CPU oracle (dcn4_oracle.c) into a shared library with gcc.

Test infrastructure only: the product library never loads the result.
Flags: -ffp-contract=off keeps every fp32 multiply and add separately
rounded (no fused multiply-add), which the oracle's position arithmetic
relies on; -fopenmp lets the outer image/row loops run on every core.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "dcn4_oracle.c")
LIBRARY = os.path.join(HERE, "liboracle_dcn4.so")

CFLAGS = ["-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
          "-fPIC", "-shared", "-Wall", "-Wextra"]


def build(source=SOURCE, output=LIBRARY, extra_flags=(), force=False):
    """Builds `source` into `output`; skips the compile when it is up to date."""
    if (not force and os.path.exists(output)
            and os.path.getmtime(output) >= os.path.getmtime(source)):
        return output
    cmd = ["gcc", *CFLAGS, *extra_flags, source, "-o", output, "-lm"]
    subprocess.run(cmd, check=True)
    return output


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
