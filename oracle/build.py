"""Compile the f64 CPU oracle (test infrastructure) with gcc.

Usage: python oracle/build.py [--mutation N] [--out PATH]

The default output is oracle/liboracle_gqa.so. A mutation build compiles a
deliberately wrong variant (ORACLE_MUTATION=N) for the mutation test only.
"""
import argparse
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gqa_oracle.cpp")
DEFAULT_OUT = os.path.join(HERE, "liboracle_gqa.so")


def build(out=DEFAULT_OUT, mutation=0, quiet=True):
    cmd = ["g++", "-std=c++17", "-O2", "-fPIC", "-shared", "-pthread",
           f"-DORACLE_MUTATION={int(mutation)}", SRC, "-o", out]
    # -O2 without -ffast-math: no reassociation of the f64 sums.
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("oracle build failed: " + " ".join(cmd))
    if not quiet:
        print(" ".join(cmd))
    return out


def needs_build(out=DEFAULT_OUT):
    return (not os.path.exists(out)) or os.path.getmtime(out) < os.path.getmtime(SRC)


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--mutation", type=int, default=0)
    ap.add_argument("--out", default=DEFAULT_OUT)
    args = ap.parse_args()
    build(args.out, args.mutation, quiet=False)
