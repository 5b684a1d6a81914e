"""The debugging aids: the debug switch (FA_DEBUG, or the pages' names for
their library's switch, FLASH_ATTN_DEBUG / FLASH_ATTENTION_DEBUG) makes every
call synchronise and return the device status itself; the checking build
(libfa_b200_checks.so, -DFA_CHECKS) checks every global-store index on the
device. No test here faults, traps or hangs the GPU: the failure that the
debug switch reports is the withheld TMA load of the timeout test, a bounded
wait that runs out."""

import ctypes
import math
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import exact_attention_151_b200 as fa
from exact_attention_151_b200.inputs import Workload, make_qkv

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_DEBUG_SCRIPT = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
import exact_attention_151_b200 as fa
from exact_attention_151_b200.inputs import Workload, make_qkv
w = Workload("dbg", B=1, N=512, H=2, D=64, seed=5)
q, k, v = (t.cuda() for t in make_qkv(w))
o = torch.empty_like(q)
lse = torch.empty((1, 2, 512), dtype=torch.float32, device="cuda")
s = torch.cuda.current_stream().cuda_stream
a = [q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), 1, 512, 2, 64, 0.125, False, fa.FA_BF16, s]
st_bad = fa.fwd_ptr(*a, wait_limit_ns=20_000_000, withhold_v_load=True)   # returned by the call itself
st_after = fa.status_sync()                                               # already read and cleared
st_good = fa.fwd_ptr(*a)
print("STATUS", st_bad, st_after, st_good, fa.status_sync())
"""


@pytest.mark.parametrize("var", ["FA_DEBUG", "FLASH_ATTN_DEBUG", "FLASH_ATTENTION_DEBUG"])
def test_debug_switch_returns_device_status_from_the_call(var):
    env = {k: v for k, v in os.environ.items() if k not in ("FA_DEBUG", "FLASH_ATTN_DEBUG", "FLASH_ATTENTION_DEBUG")}
    env[var] = "1"
    r = subprocess.run([sys.executable, "-c", _DEBUG_SCRIPT, ROOT], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    line = [x for x in r.stdout.splitlines() if x.startswith("STATUS")][-1]
    assert line.split()[1:] == [str(fa.FA_ERR_TIMEOUT), str(fa.FA_OK), str(fa.FA_OK), str(fa.FA_OK)], line
    assert "[fa] fwd D=64" in r.stderr  # the launch configuration is logged
    assert "device status 5" in r.stderr


def _fwd_gqa(lib, q, k, v, o, lse, causal):
    B, Nq, Hq, D = q.shape
    _, Nk, Hkv, _ = k.shape
    s = torch.cuda.current_stream().cuda_stream
    return lib.fa_fwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Nq, Nk, Hq, Hkv,
                          D, ctypes.c_float(1 / math.sqrt(D)), int(causal), fa._dtype_code(q), s)


def _same_bits(a, b):
    return torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8))


@pytest.mark.parametrize("B,Nq,Nk,Hq,Hkv,D,dtype,causal", [
    (2, 1000, 1000, 4, 4, 64, "fp16", True),     # ragged last tile, causal
    (1, 777, 777, 2, 2, 128, "bf16", False),
    (2, 300, 1000, 8, 2, 128, "bf16", True),     # cross lengths, grouped heads
    (2, 3, 517, 12, 3, 64, "fp16", True),        # packed heads
])
def test_checking_build_is_bit_identical_and_clean(B, Nq, Nk, Hq, Hkv, D, dtype, causal):
    chk = fa.load_checking_library()
    lib = fa.load_library()
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    g = torch.Generator().manual_seed(B * 7 + Nq + Nk)
    q = torch.randn(B, Nq, Hq, D, generator=g).to(tdt).to(DEV)
    k = torch.randn(B, Nk, Hkv, D, generator=g).to(tdt).to(DEV)
    v = torch.randn(B, Nk, Hkv, D, generator=g).to(tdt).to(DEV)
    outs = []
    for L in (lib, chk):
        o = torch.full_like(q, float("nan"))
        lse = torch.full((B, Hq, Nq), float("nan"), device=DEV)
        assert _fwd_gqa(L, q, k, v, o, lse, causal) == fa.FA_OK
        assert L.fa_status_sync(torch.cuda.current_stream().cuda_stream) == fa.FA_OK
        outs.append((o, lse))
    assert _same_bits(outs[0][0], outs[1][0]) and _same_bits(outs[0][1], outs[1][1])


def test_checking_build_splitkv_and_backward_are_bit_identical():
    chk = fa.load_checking_library()
    lib = fa.load_library()
    s = torch.cuda.current_stream().cuda_stream
    # split-KV (paired, packed heads)
    B, Nq, Nk, Hq, Hkv, D = 1, 1, 20000, 32, 8, 128
    g = torch.Generator().manual_seed(3)
    q = torch.randn(B, Nq, Hq, D, generator=g).to(torch.bfloat16).to(DEV)
    k = torch.randn(B, Nk, Hkv, D, generator=g).to(torch.bfloat16).to(DEV)
    v = torch.randn(B, Nk, Hkv, D, generator=g).to(torch.bfloat16).to(DEV)
    n, need = fa.splitkv_plan(B, Nq, Nk, Hq, D, Hkv=Hkv)
    assert n > 1
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    outs = []
    for L in (lib, chk):
        o = torch.full_like(q, float("nan"))
        lse = torch.full((B, Hq, Nq), float("nan"), device=DEV)
        st = L.fa_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Nq, Nk, Hq,
                              Hkv, D, ctypes.c_float(1 / math.sqrt(D)), 1, fa.FA_BF16, 0, ws.data_ptr(), need, s)
        assert st == fa.FA_OK and L.fa_status_sync(s) == fa.FA_OK
        outs.append((o, lse))
    assert _same_bits(outs[0][0], outs[1][0]) and _same_bits(outs[0][1], outs[1][1])
    # backward
    w = Workload("chk_bwd", B=1, N=300, H=2, D=64, causal=True, seed=9)
    q, k, v = (t.to(DEV) for t in make_qkv(w))
    o, lse = fa.fwd(q, k, v, causal=True)
    dout = torch.randn(q.shape, generator=g).to(q.dtype).to(DEV)
    need = fa.bwd_workspace_size(1, 300, 2)
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    grads = []
    for L in (lib, chk):
        dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
        st = L.fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), dout.data_ptr(),
                      dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), 1, 300, 2, 64, ctypes.c_float(w.softmax_scale), 1,
                      fa.FA_BF16, ws.data_ptr(), need, s)
        assert st == fa.FA_OK and L.fa_status_sync(s) == fa.FA_OK
        grads.append((dq, dk, dv))
    for a, b in zip(*grads):
        assert _same_bits(a, b)


def test_checking_build_reports_inconsistent_offsets():
    """Offsets in device memory are outside what the host can validate; both
    builds skip the bad sequence and report it through the status word."""
    chk = fa.load_checking_library()
    H, D = 2, 64
    g = torch.Generator().manual_seed(31)
    q = torch.randn(100, H, D, generator=g).to(torch.bfloat16).to(DEV)
    cu_q = torch.tensor([0, 60, 40, 100], dtype=torch.int32, device=DEV)
    cu_k = torch.tensor([0, 30, 60, 100], dtype=torch.int32, device=DEV)
    o = torch.full_like(q, 7.0)
    lse = torch.full((H, 100), 7.0, device=DEV)
    s = torch.cuda.current_stream().cuda_stream
    st = chk.fa_fwd_varlen(q.data_ptr(), q.data_ptr(), q.data_ptr(), o.data_ptr(), lse.data_ptr(), cu_q.data_ptr(),
                           cu_k.data_ptr(), 3, 60, 100, 100, H, H, D, ctypes.c_float(0.125), 0, fa.FA_BF16, s)
    assert st == fa.FA_OK
    assert chk.fa_status_sync(s) == fa.FA_ERR_INVALID_ARG
    assert chk.fa_status_sync(s) == fa.FA_OK
    assert np.isfinite(o[:40].float().cpu().numpy()).all()  # sequence 0 was computed
