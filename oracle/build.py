"""Build the fp64 CPU oracle (test infrastructure) into oracle/libssd_oracle.so.

Plain gcc, no fast-math: the oracle's floating-point order is the order written in
ssd_oracle.c.  `extra_defines` exists so a test can compile a deliberately wrong copy of
the oracle (a planted mistake) into a scratch directory and check that the pins catch it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ssd_oracle.c")
LIB = os.path.join(HERE, "libssd_oracle.so")


def build(out_path: str = LIB, extra_defines=(), force: bool = False) -> str:
    if (not force and os.path.exists(out_path)
            and os.path.getmtime(out_path) >= os.path.getmtime(SRC) and not extra_defines):
        return out_path
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-fno-fast-math",
           "-ffp-contract=off", "-Wall", "-Wextra", "-o", out_path + ".tmp", SRC, "-lm"]
    cmd[1:1] = ["-D" + d for d in extra_defines]
    subprocess.run(cmd, check=True)
    os.replace(out_path + ".tmp", out_path)
    return out_path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
