"""Build libmoe_b200.so in-tree for sm_100a with nvcc (no JIT, no torch extension)."""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libmoe_b200.so")
SOURCES = ["api.cu", "permute.cu", "combine.cu", "tensor_maps.cu", "grouped_ffn.cu",
           "grouped_ffn_bwd.cu", "grouped_ffn_mx.cu"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-lineinfo",
              "-gencode", "arch=compute_100a,code=sm_100a"]


def build(verbose: bool = False, extra: list[str] | None = None) -> str:
    srcs = [os.path.join(HERE, "csrc", s) for s in SOURCES]
    cmd = ["nvcc", *NVCC_FLAGS, *(extra or []), "-I", os.path.join(ROOT, "include"), *srcs,
           "-o", LIB]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(verbose=True)
