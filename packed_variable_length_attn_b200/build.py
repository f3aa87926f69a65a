"""Build the CUDA library libvarlen_attn.so in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC_DIR = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libvarlen_attn.so")
SOURCES = ["varlen_attn.cu"]
# Every header the translation unit includes (a stale library is rebuilt when
# any of them changes); checked against the csrc directory below.
HEADERS = ["attn_sm100.cuh", "attn_f32.cuh", "sched.cuh", "common.cuh", "ptx.cuh", "layout.cuh",
           "decode.cuh"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _inputs():
    # the listed files plus anything else in csrc, so a new header can never
    # leave a stale library behind
    names = set(SOURCES + HEADERS)
    names |= {f for f in os.listdir(SRC_DIR) if f.endswith((".cu", ".cuh"))}
    files = [os.path.join(SRC_DIR, f) for f in sorted(names)]
    files.append(os.path.join(ROOT, "include", "varlen_attn.h"))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-cudart", "static",
           "-I", os.path.join(ROOT, "include"), "-o", tmp]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(SRC_DIR, s) for s in SOURCES]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
