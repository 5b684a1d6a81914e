"""Failure detection without a GPU fault: a withheld TMA load makes one CTA's
bounded waits run out; the kernel gives up cleanly (TMEM freed, loads
drained), records FA_ERR_TIMEOUT in the device status word, and the next
normal call on the same GPU is correct."""

import pytest
import torch

import exact_attention_151_b200 as fa
import oracle
from exact_attention_151_b200.inputs import Workload, bits, make_qkv
from tests.parity import metrics, passes

pytestmark = pytest.mark.gpu


def test_withheld_load_reports_timeout_and_gpu_recovers():
    w = Workload("timeout", B=1, N=512, H=2, D=64, seed=5)
    q, k, v = make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.empty_like(qd)
    lse = torch.empty((1, 2, 512), dtype=torch.float32, device="cuda")
    assert fa.status_sync() == fa.FA_OK
    fa.fwd_into(qd, kd, vd, o, lse, wait_limit_ns=20_000_000, withhold_v_load=True)
    assert fa.status_sync() == fa.FA_ERR_TIMEOUT
    assert fa.status_sync() == fa.FA_OK  # the word is cleared by the read
    fa.fwd_into(qd, kd, vd, o, lse)
    assert fa.status_sync() == fa.FA_OK
    o_ref, lse_ref = oracle.attention(bits(q), bits(k), bits(v), w.softmax_scale, False, "bf16")
    m = metrics(o.cpu().double().numpy(), lse.cpu().double().numpy(), o_ref, lse_ref)
    assert passes(m), m
