"""Builds the in-tree CUDA library libw4a8.so for sm_100a with nvcc.

Usage: python -m w4a8_quantized_gemm_quantize_b200.build [--force] [--verbose] [--debug]

--debug builds libw4a8_debug.so instead: the same library compiled with
W4A8_DEBUG, whose kernels check every global store and workspace access
against its buffer's extent and report a failed check in the device error
word (W4A8_DEVERR_BOUNDS) instead of performing the access.

The shared library links the CUDA runtime statically and resolves the one
driver entry point it needs (cuTensorMapEncodeTiled) at run time, so it
loads on a machine without a GPU driver (its symbols can be inspected there)
and runs on any machine with a B200 driver.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libw4a8.so"
LIB_PATH = os.path.join(PKG_DIR, LIB_NAME)
DEBUG_LIB_PATH = os.path.join(PKG_DIR, "libw4a8_debug.so")
SOURCES = ["w4a8_api.cu"]
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found (set NVCC or put it on PATH)")


def _inputs():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh"))]
    files.append(os.path.join(INCLUDE, "w4a8.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    path = DEBUG_LIB_PATH if debug else LIB_PATH
    if not force and up_to_date(path):
        return path
    tmp = path + ".tmp"
    cmd = [
        _nvcc(), *ARCH_FLAGS, "-O3", "-std=c++17", "-lineinfo", "--shared", "-Xcompiler", "-fPIC",
        "-Xcompiler", "-fvisibility=hidden", "-cudart", "static", "-I", INCLUDE, "-I", CSRC,
        "-DW4A8_BUILD",
    ]
    if debug:
        cmd.append("-DW4A8_DEBUG")
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES] + ["-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, path)
    return path


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--debug", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose, debug=args.debug))


if __name__ == "__main__":
    main()
