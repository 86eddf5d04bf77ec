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


def build(out=LIB, verbose=False, force=False):
    if not force and not needs_build(out):
        return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    cmd = nvcc_command(out)
    res = subprocess.run(cmd, capture_output=True, text=True)
    log = os.path.join(os.path.dirname(out), "ptxas.log")
    with open(log, "w") as f:
        f.write(" ".join(cmd) + "\n" + res.stdout + res.stderr)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc build of libgqa_decode.so failed")
    if verbose:
        print(" ".join(cmd))
        print(res.stderr)
    return out


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    build(verbose=a.verbose, force=a.force)
