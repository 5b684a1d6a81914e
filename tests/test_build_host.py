"""The sm_100a build as ptxas reports it, on the CPU (nvcc cross-compiles).

The forward kernel moves registers between its warpgroups with setmaxnreg:
the control warpgroup gives some back and the two softmax warpgroups take
them. That is only safe when every thread was launched with exactly the count
the split was sized for, so the host refuses to launch a build whose count
differs (FA_ERR_UNSUPPORTED). This test compiles the sources the way the build
does, with ptxas reporting, and checks every forward instantiation against
the count in the kernel header. It also checks that the split fits the pool
the launch provides, so that a source change breaking either is caught here
rather than on a GPU.
"""

import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_attention_151_b200", "csrc")


def _header_constant(name):
    src = open(os.path.join(CSRC, "fa_fwd_kernel.cuh")).read()
    m = re.search(rf"constexpr (?:uint32_t|int) {name} = (\d+);", src)
    assert m, name
    return int(m.group(1))


@pytest.fixture(scope="module")
def ptxas_report(tmp_path_factory):
    from exact_attention_151_b200 import build

    try:
        nvcc = build.nvcc_path()
    except RuntimeError:
        pytest.skip("nvcc not available")
    out = tmp_path_factory.mktemp("ptxas") / "lib.so"
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17", "-Xcompiler",
           "-fPIC", "-shared", "--cudart", "static", f"-I{os.path.join(ROOT, 'include')}", f"-I{CSRC}",
           "-Xptxas=-v", "-o", str(out), os.path.join(CSRC, "fa_fwd.cu")]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    regs, spills, cur = {}, {}, None
    for line in r.stderr.splitlines():
        m = re.search(r"Compiling entry function '(\S+)'", line)
        if m:
            cur = m.group(1)
            continue
        m = re.search(r"(\d+) bytes spill stores", line)
        if m and cur:
            spills[cur] = int(m.group(1))
        m = re.search(r"Used (\d+) registers", line)
        if m and cur:
            regs[cur] = int(m.group(1))
            cur = None
    return regs, spills


def test_every_forward_instantiation_has_the_launch_register_count(ptxas_report):
    launch = _header_constant("kLaunchRegs")
    regs, _ = ptxas_report
    fwd = {k: v for k, v in regs.items() if "fa_fwd_kernel" in k}
    # D in {64, 128} x {bf16, fp16} x {unpaired, paired split-KV}
    assert len(fwd) == 8, sorted(fwd)
    assert all(v == launch for v in fwd.values()), fwd


def test_register_split_fits_the_launch_pool():
    threads = _header_constant("kThreads")
    launch = _header_constant("kLaunchRegs")
    soft = _header_constant("kSoftmaxRegs")
    ctrl = _header_constant("kControlRegs")
    assert threads % 128 == 0
    n_groups = threads // 128
    assert 128 * ((n_groups - 1) * soft + ctrl) <= threads * launch
    # setmaxnreg counts are multiples of 8 within [24, 256]
    for r in (soft, ctrl):
        assert r % 8 == 0 and 24 <= r <= 256
    # the launch count is what the register file allows at one CTA per SM
    assert threads * launch <= 65536


def test_backward_kernels_compile_without_spills(ptxas_report):
    regs, spills = ptxas_report
    bwd = {k: spills.get(k) for k in regs if "fa_bwd_" in k}
    # dQ and dK/dV kernels, preprocess and packed preprocess, for D in {64, 128} x {bf16, fp16}
    assert len(bwd) == 16, sorted(bwd)
    assert all(v == 0 for v in bwd.values()), bwd
