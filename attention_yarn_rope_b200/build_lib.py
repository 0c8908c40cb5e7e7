"""Builds libgptoss_attn.so in-tree with nvcc for sm_100a.

Usage: ``python -m attention_yarn_rope_b200.build_lib [--verbose-ptxas]``.
The library is one translation unit (``csrc/gptoss_lib.cu``) linked against
the static CUDA runtime, so it needs no libcudart at load time.  The same
sources built with ``GPTOSS_DEBUG_CHECKS`` give libgptoss_attn_debug.so,
whose kernels range-check their computed indices (a bad one is recorded in
the device status word and the access skipped).
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "gptoss_lib.cu")
OUT = os.path.join(PKG, "libgptoss_attn.so")
OUT_DEBUG = os.path.join(PKG, "libgptoss_attn_debug.so")
DEPS = [os.path.join(PKG, "csrc", f) for f in os.listdir(os.path.join(PKG, "csrc"))] + [
    os.path.join(ROOT, "include", "gptoss.h")
]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def up_to_date(out: str = OUT) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(d) <= t for d in DEPS if os.path.exists(d))


def build(force: bool = False, ptxas_verbose: bool = False, debug_checks: bool = False) -> str:
    out = OUT_DEBUG if debug_checks else OUT
    if not force and up_to_date(out):
        return out
    cmd = [
        nvcc_path(),
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-O3", "-lineinfo", "-std=c++17",
        "-Xptxas=-O3",
        "-Xcompiler", "-fPIC",
        "-shared", "-cudart", "static",
        "-I", os.path.join(ROOT, "include"),
        "-o", out + ".tmp", SRC,
    ]
    if debug_checks:
        cmd.insert(1, "-DGPTOSS_DEBUG_CHECKS")
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    proc = subprocess.run(cmd, capture_output=True, text=True)
    if proc.returncode != 0:
        sys.stderr.write(proc.stdout + proc.stderr)
        raise RuntimeError("nvcc failed building libgptoss_attn.so")
    if ptxas_verbose:
        sys.stderr.write(proc.stderr)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--debug-checks", action="store_true", help="build libgptoss_attn_debug.so")
    a = ap.parse_args()
    print(build(force=a.force, ptxas_verbose=a.verbose_ptxas, debug_checks=a.debug_checks))
