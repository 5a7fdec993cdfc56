"""Compile the C oracle into ``oracle/liboracle.so`` with gcc.

Test infrastructure only.  No -ffast-math and no FMA contraction, so every
fp32/fp64 operation is the plain IEEE one written in the source; no -march so
the library runs on any x86-64 host.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "pa_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False, out: str = LIB, mutation: int = 0) -> str:
    """Build the oracle library at ``out``.  ``mutation`` > 0 plants one of the
    deliberate mistakes the pin tests must catch (never used outside tests)."""
    if (not force and mutation == 0 and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(SRC)):
        return out
    cmd = [
        "gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
        "-fPIC", "-shared", "-Wall", "-Wextra", f"-DORACLE_MUTATION={int(mutation)}",
        "-o", out + ".tmp", SRC, "-lm",
    ]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force=True))
