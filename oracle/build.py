"""Build the float64 CPU oracle (test infrastructure only) with the host C compiler.

    python oracle/build.py

Produces oracle/libspattn_oracle.so next to this file.  No CUDA header or
source is involved; the oracle shares nothing with the CUDA library.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "spattn_oracle.c")
LIB = os.path.join(HERE, "libspattn_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    # -O2 without fast-math: IEEE semantics (NaN, -inf, exact comparisons) are
    # part of the definition.  OpenMP parallelises over independent
    # (request, head) units only; a compiler without it builds a serial oracle.
    base = ["-std=c11", "-O2", "-ffp-contract=off", "-fPIC", "-shared", "-Wall", "-o", LIB + ".tmp", SRC, "-lm"]
    tried = []
    for cc in ("/usr/bin/gcc", "gcc", os.environ.get("CC", "cc")):
        for omp in (["-fopenmp"], []):
            cmd = [cc] + omp + base
            try:
                r = subprocess.run(cmd, capture_output=True, text=True)
            except OSError as e:            # compiler not present
                tried.append((cmd, str(e)))
                r = subprocess.CompletedProcess(cmd, 127)
                continue
            tried.append((cmd, r.stderr[-400:]))
            if r.returncode == 0:
                break
        if r.returncode == 0:
            break
    else:
        raise RuntimeError("cannot build the oracle: " + repr(tried))
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
