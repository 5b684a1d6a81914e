"""Build the in-tree CUDA library ``libfa_b200.so`` for sm_100a with nvcc.

    python -m exact_attention_151_b200.build [--verbose-ptxas] [--checks]

``--checks`` builds ``libfa_b200_checks.so`` instead: the same sources with
-DFA_CHECKS, whose kernels check every global-store index on the device and
report a failure through the status word (a debugging aid; slower).

The library is compiled for sm_100a only (tcgen05 / TMA / Tensor Memory), with
the CUDA runtime linked statically so the shared object loads on a machine
without a GPU (symbol checks) and on a B200 host alike.
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
CHECKS_LIB_PATH = os.path.join(HERE, "libfa_b200_checks.so")
SOURCES = [os.path.join(CSRC, "fa_fwd.cu")]
HEADERS = [os.path.join(CSRC, "sm100.cuh"), os.path.join(CSRC, "fa_fwd_kernel.cuh"), os.path.join(CSRC, "fa_bwd_kernel.cuh"),
           os.path.join(INCLUDE, "fa.h")]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; the CUDA toolkit is required to build the library")


def _stale(path: str) -> bool:
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    return any(os.path.getmtime(p) > t for p in SOURCES + HEADERS + [__file__])


def build(force: bool = False, ptxas_verbose: bool = False, checks: bool = False) -> str:
    path = CHECKS_LIB_PATH if checks else LIB_PATH
    if not (force or ptxas_verbose or _stale(path)):
        return path
    cmd = [
        nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
        "-Xcompiler", "-fPIC", "-shared", "--cudart", "static", f"-I{INCLUDE}", f"-I{CSRC}",
        "-o", path + ".tmp", *SOURCES,
    ]
    if checks:
        cmd.insert(1, "-DFA_CHECKS")
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(path + ".tmp", path)
    return path


if __name__ == "__main__":
    print(build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv, checks="--checks" in sys.argv))
