"""Build the CPU oracle shared library (test infrastructure only).

The oracle is plain C compiled with strict IEEE single-precision semantics:
no contraction into FMA, no fast-math, SSE arithmetic (no x87 excess
precision).  OpenMP only splits independent blocks across host threads.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "nvfp4_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = [
    "-O2", "-std=c11", "-fPIC", "-shared",
    "-ffp-contract=off", "-fno-fast-math", "-fexcess-precision=standard",
    "-mfpmath=sse", "-msse2", "-fopenmp", "-Wall", "-Wextra",
]


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source if it is missing or stale."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    cmd = ["gcc", *CFLAGS, SRC, "-o", LIB + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


def build_variant(source: str, out_dir: str, name: str = "liboracle_variant.so") -> str:
    """Compile a modified copy of the oracle source (tests that plant a
    mistake in the oracle and check that a pin catches it) into out_dir."""
    src = os.path.join(out_dir, name.replace(".so", ".c"))
    with open(src, "w") as f:
        f.write(source)
    lib = os.path.join(out_dir, name)
    subprocess.run(["gcc", *CFLAGS, src, "-o", lib, "-lm"], check=True)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
