"""Builds libfia.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python paged_attention_02_b200/build.py [--force] [--verbose] [--ptxas-info]

Run it as a script (or load it by file path, as ``load_builder()`` in
``__graft_entry__`` does): importing it through the package would first load
the library it is meant to build.

Static CUDA runtime, no libcuda link dependency (the driver entry point for
TMA descriptor encoding is looked up at run time), so the library loads on a
machine without a GPU; every compute entry point then reports FIA_ERR_CUDA.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
REPO = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
LIB_PATH = os.path.join(PKG_DIR, "libfia.so")
SOURCES = ["fia_host.cu", "decode_kernel.cu", "prefill_kernel.cu"]
HEADERS = ["fia_device.cuh", "fia_plan.h", "prefill_common.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    p = shutil.which("nvcc")
    if p:
        return p
    p = "/usr/local/cuda/bin/nvcc"
    if os.path.exists(p):
        return p
    raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libfia.so")


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(REPO, "include", "fia.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    if not force and up_to_date():
        return LIB_PATH
    tmp = LIB_PATH + ".tmp%d" % os.getpid()
    cmd = [nvcc_path(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "--shared",
           "-Xcompiler", "-fPIC,-fvisibility=hidden", "-cudart", "static",
           "--expt-relaxed-constexpr", "-I", os.path.join(REPO, "include"),
           "-o", tmp] + [os.path.join(CSRC, f) for f in SOURCES]
    if ptxas_info:
        cmd.insert(1, "-Xptxas=-v")
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if ptxas_info or verbose:
        sys.stdout.write(r.stdout)
        sys.stdout.write(r.stderr)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, ptxas_info=a.ptxas_info))
