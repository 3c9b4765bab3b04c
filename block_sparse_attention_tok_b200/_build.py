"""Builds libsparstar.so (the C-ABI library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libsparstar.so"
LIB_PATH = os.path.join(PKG_DIR, LIB_NAME)
SOURCES = ["sparstar.cu"]
DEPENDS = ["sparstar.cu", "ptx.cuh", "select.cuh", "attn_sm100.cuh", "mass_sm100.cuh"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def nvcc_command(out_path: str = LIB_PATH, extra=()) -> list:
    return [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
            "-shared", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-o", out_path,
            *[os.path.join(CSRC, s) for s in SOURCES], *extra]


def up_to_date(out_path: str = LIB_PATH) -> bool:
    if not os.path.exists(out_path):
        return False
    t = os.path.getmtime(out_path)
    deps = [os.path.join(CSRC, s) for s in DEPENDS] + [os.path.join(INCLUDE, "sparstar.h")]
    return all(os.path.getmtime(p) <= t for p in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB_PATH
    cmd = nvcc_command()
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    tmp = LIB_PATH + ".tmp"
    cmd[cmd.index("-o") + 1] = tmp
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
