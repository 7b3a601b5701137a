"""Build the CUDA library ``libcoli_moe.so`` in-tree for sm_100a."""
from __future__ import annotations

import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(HERE, "libcoli_moe.so")

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
    "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared", "--expt-relaxed-constexpr",
]


def build(verbose: bool = False, extra: list[str] | None = None) -> str:
    """COLI_TC_TRACE=1 in the environment builds the profiling variant whose
    tensor-core kernels record a block timeline into the trace buffer."""
    srcs = sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))
    flags = list(extra or [])
    if os.environ.get("COLI_TC_TRACE") == "1":
        flags.append("-DCOLI_TC_TRACE=1")
    cmd = ["nvcc", *NVCC_FLAGS, *flags, "-o", SO, *srcs]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    return SO


if __name__ == "__main__":
    build(verbose=True)
