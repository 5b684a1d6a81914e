"""Build the in-tree CUDA library ``libfa_b200.so`` for sm_100a with nvcc.

    python -m exact_attention_151_b200.build [--verbose-ptxas]

The library is compiled for sm_100a only (tcgen05 / TMA / Tensor Memory), with
the CUDA runtime linked statically so the shared object loads on a machine
without a GPU (symbol checks) and on the GPU machine alike.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libfa_b200.so"
LIB_PATH = os.path.join(HERE, LIB_NAME)
SOURCES = [os.path.join(CSRC, "fa_fwd.cu")]
HEADERS = [os.path.join(CSRC, "sm100.cuh"), os.path.join(CSRC, "fa_fwd_kernel.cuh"), os.path.join(CSRC, "fa_bwd_kernel.cuh"),
           os.path.join(INCLUDE, "fa.h")]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; the CUDA toolkit is required to build the library")


def _stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    return any(os.path.getmtime(p) > t for p in SOURCES + HEADERS + [__file__])


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    if not (force or ptxas_verbose or _stale()):
        return LIB_PATH
    cmd = [
        nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
        "-Xcompiler", "-fPIC", "-shared", "--cudart", "static", f"-I{INCLUDE}", f"-I{CSRC}",
        "-o", LIB_PATH + ".tmp", *SOURCES,
    ]
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(LIB_PATH + ".tmp", LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv))
