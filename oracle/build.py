"""Build the float64 CPU oracle (test infrastructure only).

    python oracle/build.py            # -> oracle/liboracle.so
    python oracle/build.py --mutant 3 --out /tmp/liboracle_m3.so

The mutant switch plants one deliberate mistake (see oracle.c) and is used
only by the tests that show each pin catches it.
"""
import argparse
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
DEFAULT_OUT = os.path.join(HERE, "liboracle.so")


def build(out: str = DEFAULT_OUT, mutant: int = 0, quiet: bool = True) -> str:
    """Compile oracle.c with gcc (-O2, OpenMP, plain IEEE float64 math)."""
    cmd = [
        "gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
        "-fno-fast-math", "-ffp-contract=off",
        f"-DAGREF_MUTANT={int(mutant)}", SRC, "-o", out, "-lm",
    ]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("oracle build failed:\n" + res.stdout + res.stderr)
    if not quiet:
        print(" ".join(cmd))
    return out


def ensure_built() -> str:
    """Build liboracle.so if it is missing or older than its source."""
    if (not os.path.exists(DEFAULT_OUT)
            or os.path.getmtime(DEFAULT_OUT) < os.path.getmtime(SRC)):
        build(DEFAULT_OUT)
    return DEFAULT_OUT


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--out", default=DEFAULT_OUT)
    ap.add_argument("--mutant", type=int, default=0)
    a = ap.parse_args()
    print(build(a.out, a.mutant, quiet=False))
    sys.exit(0)
