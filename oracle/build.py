"""Compile the fp64 CPU oracle (test infrastructure) into oracle/_build/libgdr_oracle.so.

Plain gcc, -O2, no -ffast-math (IEEE semantics kept), OpenMP over independent head-units.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gdr_oracle.c")
OUT_DIR = os.path.join(HERE, "_build")
OUT = os.path.join(OUT_DIR, "libgdr_oracle.so")


def build(src=SRC, out=OUT, extra_flags=(), quiet=True):
    """Compile ``src`` into the shared library ``out``; returns ``out``."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC",
           "-shared", "-std=c99", *extra_flags, src, "-o", out, "-lm"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"oracle build failed: {' '.join(cmd)}\n{res.stderr}")
    if not quiet and res.stderr:
        sys.stderr.write(res.stderr)
    return out


def needs_build(out=OUT, src=SRC):
    return (not os.path.exists(out)) or os.path.getmtime(out) < os.path.getmtime(src)


if __name__ == "__main__":
    print(build(quiet=False))
