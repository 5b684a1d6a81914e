"""GPU parity of the generalised forward: grouped-query heads, queries and
keys of different lengths (bottom-right causal), and packed sequences of
different lengths, against the oracle's packed-sequence form."""

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


def _randn(shape, seed, dtype=torch.bfloat16, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(dtype)


def _check(o, lse, o_ref, lse_ref):
    """Parity with the -inf LSE of key-less rows compared exactly."""
    lse = np.asarray(lse, dtype=np.float64)
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty)
    m = metrics(o, np.where(empty, 0.0, lse), o_ref, np.where(empty, 0.0, lse_ref))
    assert passes(m), m
    return m


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(256, 256), (300, 300), (128, 1000), (1000, 128), (513, 700), (700, 513),
                                   (1, 300), (300, 1), (64, 0)])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (4, 1)])
def test_dense_gqa_cross_lengths(Nq, Nk, Hq, Hkv, causal):
    B, D = 2, 128
    seed = Nq * 7 + Nk + Hq * 3 + Hkv
    q = _randn((B, Nq, Hq, D), seed)
    k = _randn((B, Nk, Hkv, D), seed + 1)
    v = _randn((B, Nk, Hkv, D), seed + 2)
    o, lse = fa.fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal)
    assert fa.status_sync() == fa.FA_OK
    cu_q, cu_k = np.arange(B + 1) * Nq, np.arange(B + 1) * Nk
    o_ref, lse_ref = oracle.attention_varlen(bits(q.reshape(B * Nq, Hq, D)), bits(k.reshape(B * Nk, Hkv, D)),
                                             bits(v.reshape(B * Nk, Hkv, D)), cu_q, cu_k, 1 / math.sqrt(D), causal,
                                             "bf16")
    _check(o.cpu().double().reshape(B * Nq, Hq, D).numpy(),
           lse.cpu().permute(1, 0, 2).reshape(Hq, B * Nq).numpy(), o_ref, lse_ref)


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("fp16", 64)])
@pytest.mark.parametrize("causal", [False, True])
def test_packed_sequences(dtype, D, causal):
    lens_q = [1, 0, 257, 128, 700, 33, 1024]
    lens_k = [5, 3, 257, 300, 700, 1, 1024]
    Hq, Hkv = 8, 2
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    q = _randn((sum(lens_q), Hq, D), 11, tdt)
    k = _randn((sum(lens_k), Hkv, D), 12, tdt)
    v = _randn((sum(lens_k), Hkv, D), 13, tdt)
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    o = torch.full_like(q.to(DEV), float("nan"))
    lse = torch.full((Hq, sum(lens_q)), float("nan"), device=DEV)
    fa.fwd_varlen(q.to(DEV), k.to(DEV), v.to(DEV), torch.from_numpy(cu_q).to(DEV), torch.from_numpy(cu_k).to(DEV),
                  max(lens_q), causal=causal, o=o, lse=lse)
    assert fa.status_sync() == fa.FA_OK
    o_ref, lse_ref = oracle.attention_varlen(bits(q), bits(k), bits(v), cu_q, cu_k, 1 / math.sqrt(D), causal, dtype)
    _check(o.cpu().double().numpy(), lse.cpu().numpy(), o_ref, lse_ref)


def test_packed_equals_dense_bitwise():
    """Equal-length packed sequences give exactly the dense call's bits."""
    B, N, H, D = 3, 300, 4, 128
    q, k, v = (_randn((B, N, H, D), s) for s in (21, 22, 23))
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o1, l1 = fa.fwd(qd, kd, vd, causal=True)
    cu = torch.arange(B + 1, dtype=torch.int32, device=DEV) * N
    o2, l2 = fa.fwd_varlen(qd.reshape(B * N, H, D), kd.reshape(B * N, H, D), vd.reshape(B * N, H, D), cu, cu, N,
                           causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1.reshape(B * N, H, D).view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1.permute(1, 0, 2).reshape(H, B * N).view(torch.int32), l2.view(torch.int32))


def test_inconsistent_offsets_are_reported_and_skipped():
    H, D = 2, 64
    q = _randn((100, H, D), 31).to(DEV)
    k = _randn((100, H, D), 32).to(DEV)
    cu_q = torch.tensor([0, 60, 40, 100], dtype=torch.int32, device=DEV)  # decreasing: sequence 1 is invalid
    cu_k = torch.tensor([0, 30, 60, 100], dtype=torch.int32, device=DEV)
    o = torch.full_like(q, 7.0)
    lse = torch.full((H, 100), 7.0, device=DEV)
    fa.fwd_varlen(q, k, k, cu_q, cu_k, 60, o=o, lse=lse)
    assert fa.status_sync() == fa.FA_ERR_INVALID_ARG
    assert fa.status_sync() == fa.FA_OK
    # sequence 0 (rows 0..59) was valid and computed; nothing was written for the bad one
    assert bool(torch.isfinite(o[:60]).all()) and not bool((o[:60] == 7.0).all())
    # a length beyond max_seqlen_q is also rejected
    cu_q2 = torch.tensor([0, 10, 100], dtype=torch.int32, device=DEV)
    cu_k2 = torch.tensor([0, 10, 100], dtype=torch.int32, device=DEV)
    fa.fwd_varlen(q, k, k, cu_q2, cu_k2, 50, o=o, lse=lse)
    assert fa.status_sync() == fa.FA_ERR_INVALID_ARG


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,Nq,Nk,Hq,Hkv,D,dtype", [
    (2, 1, 300, 8, 2, 128, "bf16"),     # decode, 4 heads per K/V head
    (1, 16, 1000, 32, 4, 128, "bf16"),  # 16 x 8 = 128 rows: a full packed tile
    (3, 3, 517, 12, 3, 64, "fp16"),     # ragged: 12 rows, bottom-right causal with several queries
    (1, 2, 64, 64, 1, 128, "bf16"),     # 64 heads on one K/V head, fewer keys than a tile
    (2, 5, 0, 8, 4, 64, "bf16"),        # no keys: O = 0, LSE = -inf
])
def test_packed_heads(B, Nq, Nk, Hq, Hkv, D, dtype, causal):
    """Nq * (Hq / Hkv) <= 128: the query heads sharing a K/V head are packed into one tile."""
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    seed = B * 1000 + Nq * 31 + Nk + Hq
    q = _randn((B, Nq, Hq, D), seed, tdt)
    k = _randn((B, Nk, Hkv, D), seed + 1, tdt)
    v = _randn((B, Nk, Hkv, D), seed + 2, tdt)
    o, lse = fa.fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal)
    assert fa.status_sync() == fa.FA_OK
    cu_q, cu_k = np.arange(B + 1) * Nq, np.arange(B + 1) * Nk
    o_ref, lse_ref = oracle.attention_varlen(bits(q.reshape(B * Nq, Hq, D)), bits(k.reshape(B * Nk, Hkv, D)),
                                             bits(v.reshape(B * Nk, Hkv, D)), cu_q, cu_k, 1 / math.sqrt(D), causal,
                                             dtype)
    lse_g = lse.cpu().permute(1, 0, 2).reshape(Hq, B * Nq).numpy()
    finite = np.isfinite(lse_ref)
    assert np.all(np.isneginf(lse_g[~finite]))
    _check(o.cpu().double().reshape(B * Nq, Hq, D).numpy(), np.where(finite, lse_g, 0.0), o_ref,
           np.where(finite, lse_ref, 0.0))
