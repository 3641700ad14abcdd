"""Build the qt2 CUDA library in-tree: nvfp4_quantized_b200/libqt2.so (sm_100a only), and with
--checked its checked build libqt2_checked.so (-DQT2_CHECKED: every kernel store checked
against its output array, see include/qt2.h).

    python -m nvfp4_quantized_b200.build [--force] [--verbose] [--checked]

nvcc cross-compiles without a GPU.  --fmad=false keeps every floating-point expression of
the quantizers an individually rounded IEEE operation (they also use explicit _rn intrinsics).
"""
from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libqt2.so")
LIB_CHECKED = os.path.join(PKG, "libqt2_checked.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(CSRC, "*.h")) + [os.path.join(INCLUDE, "qt2.h")])


def nvcc_cmd(out: str, verbose: bool = False, checked: bool = False):
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "--fmad=false", "-std=c++17",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-shared", "-I", INCLUDE, "-I", CSRC,
           "-o", out, os.path.join(CSRC, "qt2_lib.cu"), os.path.join(CSRC, "qt2_noalloc.cu")]
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    if checked:
        cmd[1:1] = ["-DQT2_CHECKED"]
    return cmd


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    lib = LIB_CHECKED if checked else LIB
    newest = max(os.path.getmtime(p) for p in sources())
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= newest and not verbose:
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    res = subprocess.run(nvcc_cmd(tmp, verbose, checked), capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(lib)}")
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--checked", action="store_true", help="build libqt2_checked.so instead")
    a = ap.parse_args()
    print(build(a.force, a.verbose, a.checked))
