"""GPU parity of the split-KV forward (keys cut into ranges, partial results
merged by a second kernel) against the oracle, on decode-like shapes."""

import math

import numpy as np
import pytest
import torch

import exact_attention_151_b200 as fa
import oracle
from exact_attention_151_b200.inputs import bits
from tests.parity import metrics, passes

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _randn(shape, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(dtype)


def _oracle_dense(q, k, v, causal, dtype):
    B, Nq, Hq, D = q.shape
    _, Nk, Hkv, _ = k.shape
    o, lse = oracle.attention_varlen(bits(q.reshape(B * Nq, Hq, D)), bits(k.reshape(B * Nk, Hkv, D)),
                                     bits(v.reshape(B * Nk, Hkv, D)), np.arange(B + 1) * Nq, np.arange(B + 1) * Nk,
                                     1 / math.sqrt(D), causal, dtype)
    return o.reshape(B, Nq, Hq, D), lse.reshape(Hq, B, Nq).transpose(1, 0, 2)


def _check(o, lse, o_ref, lse_ref):
    lse = lse.cpu().double().numpy()
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty)
    m = metrics(o.cpu().double().numpy(), np.where(empty, 0.0, lse), o_ref, np.where(empty, 0.0, lse_ref))
    assert passes(m), m


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,Nq,Nk,Hq,Hkv,D,dtype,splits", [
    (1, 1, 4096, 32, 8, 128, "bf16", 0),
    (2, 1, 1000, 8, 1, 128, "bf16", 0),
    (1, 16, 8192, 8, 2, 128, "bf16", 0),
    (1, 128, 3000, 4, 4, 64, "fp16", 0),
    (1, 300, 2048, 2, 2, 128, "bf16", 3),
    (1, 1, 777, 4, 4, 64, "bf16", 64),
    (1, 4, 129, 2, 1, 128, "bf16", 2),
    # packed heads pair two key ranges per CTA: an odd count (the last CTA's
    # second range is empty), a shorter second range, ragged last tiles
    (1, 1, 3000, 8, 2, 128, "bf16", 5),
    (1, 2, 1100, 16, 4, 64, "fp16", 3),
    (1, 1, 300, 4, 1, 128, "bf16", 3),
    (1, 1, 850, 8, 2, 128, "bf16", 4),
    (2, 3, 700, 8, 2, 64, "bf16", 0),
])
def test_splitkv_matches_oracle(B, Nq, Nk, Hq, Hkv, D, dtype, splits, causal):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    seed = Nq * 13 + Nk + Hq
    q, k, v = _randn((B, Nq, Hq, D), seed, tdt), _randn((B, Nk, Hkv, D), seed + 1, tdt), _randn((B, Nk, Hkv, D), seed + 2, tdt)
    n, _ = fa.splitkv_plan(B, Nq, Nk, Hq, D, splits, Hkv=Hkv)
    assert n > 1  # these shapes are meant to split
    o, lse = fa.fwd_splitkv(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, num_splits=splits)
    assert fa.status_sync() == fa.FA_OK
    _check(o, lse, *_oracle_dense(q, k, v, causal, dtype))


def test_splitkv_close_to_unsplit_and_deterministic():
    B, Nq, Nk, Hq, Hkv, D = 1, 64, 8192, 8, 8, 128
    q, k, v = (_randn(s, i).to(DEV) for i, s in enumerate([(B, Nq, Hq, D), (B, Nk, Hkv, D), (B, Nk, Hkv, D)]))
    o1, l1 = fa.fwd(q, k, v, causal=True)
    o2, l2 = fa.fwd_splitkv(q, k, v, causal=True)
    o3, l3 = fa.fwd_splitkv(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 1e-2
    assert (l1 - l2).abs().max().item() <= 1e-3
    assert torch.equal(o2.view(torch.int16), o3.view(torch.int16)) and torch.equal(l2, l3)


def test_splitkv_rejects_small_workspace():
    B, Nq, Nk, Hq, D = 1, 1, 4096, 32, 128
    q = _randn((B, Nq, Hq, D), 1).to(DEV)
    k = _randn((B, Nk, Hq, D), 2).to(DEV)
    n, need = fa.splitkv_plan(B, Nq, Nk, Hq, D)
    assert n > 1 and need > 0
    ws = torch.empty(need - 256, dtype=torch.uint8, device=DEV)
    with pytest.raises(fa.FaError) as e:
        fa.fwd_splitkv(q, k, k, workspace=ws)
    assert e.value.code == fa.FA_ERR_INVALID_ARG
