"""Build the CUDA library libgqa_decode.so in-tree for sm_100a.

Usage: python -m gqa_decode_attention_attend_b200.build [--verbose]

The library links the CUDA runtime statically, so loading it needs no
libcudart on the library path (and loads, without running kernels, on a host
with no GPU). The driver API is reached through cudaGetDriverEntryPoint.
"""
import argparse
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libgqa_decode.so")
# The same sources with test-only hooks compiled in (GQA_TEST_HOOKS); only
# tests load it.
TEST_LIB = os.path.join(LIBDIR, "libgqa_decode_test.so")
SOURCES = [os.path.join(CSRC, "gqa_decode.cu")]
HEADERS = sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")) + [
    os.path.join(ROOT, "include", "gqa_decode.h")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_command(out=LIB, extra=()):
    return [NVCC, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
            "-shared", "--cudart", "static", f"-I{os.path.join(ROOT, 'include')}",
            "-Xptxas", "-v", *extra, *SOURCES, "-o", out, "-lrt", "-ldl", "-lpthread"]


def needs_build(out=LIB):
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS)


def _start(out, extra=()):
    os.makedirs(os.path.dirname(out), exist_ok=True)
    cmd = nvcc_command(out, extra)
    return cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)


def _finish(out, cmd, proc, verbose):
    stdout, stderr = proc.communicate()
    log = os.path.join(os.path.dirname(out), os.path.basename(out) + ".ptxas.log")
    with open(log, "w") as f:
        f.write(" ".join(cmd) + "\n" + stdout + stderr)
    if proc.returncode != 0:
        sys.stderr.write(stdout + stderr)
        raise RuntimeError(f"nvcc build of {os.path.basename(out)} failed")
    if verbose:
        print(" ".join(cmd))
        print(stderr)
    return out


def build(out=LIB, verbose=False, force=False, test_lib=False):
    """Build the library (and, with test_lib, its test copy alongside, the two
    nvcc runs in parallel) unless it is newer than every source."""
    jobs = []
    if force or needs_build(out):
        jobs.append((out, *_start(out)))
    if test_lib and (force or needs_build(TEST_LIB)):
        jobs.append((TEST_LIB, *_start(TEST_LIB, ("-DGQA_TEST_HOOKS",))))
    for o, cmd, proc in jobs:
        _finish(o, cmd, proc, verbose)
    return out


def build_test_lib(verbose=False):
    if needs_build(TEST_LIB):
        proc = _start(TEST_LIB, ("-DGQA_TEST_HOOKS",))
        _finish(TEST_LIB, *proc, verbose)
    return TEST_LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--test-lib", action="store_true", help="also build the test copy")
    a = ap.parse_args()
    build(verbose=a.verbose, force=a.force, test_lib=a.test_lib)
