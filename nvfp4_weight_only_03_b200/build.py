"""Build libnvfp4gemv.so in-tree (nvcc, sm_100a only)."""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRCS = [os.path.join(HERE, "csrc", "nvfp4_gemv.cu"), os.path.join(HERE, "csrc", "nvfp4_gemv_tc.cu")]
HDRS = [os.path.join(ROOT, "include", "nvfp4.h"), os.path.join(HERE, "csrc", "nvfp4_tc.h"),
        os.path.join(HERE, "csrc", "nvfp4_prologue.h")]
LIB = os.path.join(HERE, "libnvfp4gemv.so")

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def build(force: bool = False, verbose: bool = False) -> str:
    newest = max(os.path.getmtime(f) for f in SRCS + HDRS)
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < newest:
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [nvcc(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), *SRCS, "-o", tmp]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose=True))
