"""Build libtq4.so in-tree with nvcc for sm_100a (B200).

    python -m compressed_paged_kv_tq4_b200.build [--force] [--verbose]

The library is two translation units: csrc/tq4_api.cu (the C ABI of the
kernels, which includes the kernel headers) and csrc/tq4_pages.cpp (the host
page pool). The shared object lands next to this file so that it travels with
the source tree; it is rebuilt when any source or the public header is newer.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libtq4.so")
SOURCES = [os.path.join(HERE, "csrc", "tq4_api.cu"), os.path.join(HERE, "csrc", "tq4_pages.cpp")]
ARCH = "-gencode=arch=compute_100a,code=sm_100a"


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; the TQ4 library needs the CUDA toolkit to build")
    return cand


def _inputs():
    return (glob.glob(os.path.join(HERE, "csrc", "*")) + glob.glob(os.path.join(ROOT, "include", "*.h")) +
            [os.path.abspath(__file__)])


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in _inputs())


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    if not force and not needs_build():
        return LIB
    cmd = [_nvcc(), ARCH, "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
           "-Xcompiler", "-fPIC,-O3", "-shared", "-I", os.path.join(ROOT, "include"),
           "-o", LIB + ".tmp", *SOURCES, *extra]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed with exit code {res.returncode}")
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
