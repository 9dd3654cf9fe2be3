"""Build the CPU oracle (test infrastructure) into oracle/libq8oracle.so with gcc.

Flags keep fp32 steps IEEE and unfused: no fast-math, no contraction."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "libq8oracle.so")
SRC = os.path.join(HERE, "q8_oracle.c")
CFLAGS = ["-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
          "-fPIC", "-shared", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile the oracle if the library is missing or older than its sources."""
    srcs = [SRC, os.path.join(HERE, "q8_oracle.h")]
    if not force and os.path.exists(LIB):
        if os.path.getmtime(LIB) >= max(os.path.getmtime(s) for s in srcs):
            return LIB
    tmp = LIB + ".tmp"
    subprocess.check_call(["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"])
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
