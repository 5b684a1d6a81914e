"""The split-KV entry point that allocates nothing (fa_fwd_splitkv_noalloc).

Some callers must not allocate device memory on the call path (their GPU
memory is reserved up front by another allocator, or they cannot handle an
out-of-memory failure mid-request); this entry point keeps its partial
results in a scratch buffer compiled into the library instead of a caller
workspace. The tests call it through the C ABI twice in a row (the scratch
keeps the previous call's contents) and compare each result element by
element with the fp64 oracle, at the tolerances used throughout the tests,
and with the workspace entry point fa_fwd_splitkv. They cover the paired
split-KV path (grouped heads packed into one tile), the unpaired one (one
query head per K/V head), and a size whose automatic range count has to fall
back to a smaller one so that the partial results fit the scratch; and they
check that free device memory is the same before and after a call. The file
sits last in collection order and depends on no other test.
"""

import ctypes
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


def _inputs(seed, B, Nq, Nk, Hq, Hkv, D):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Nq, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(B, Nk, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Nk, Hkv, D, generator=g).to(torch.bfloat16)
    return q, k, v


def _noalloc_abi(q, k, v, o, lse, causal, num_splits=0):
    B, Nq, Hq, D = q.shape
    _, Nk, Hkv, _ = k.shape
    stream = torch.cuda.current_stream().cuda_stream
    return fa.load_library().fa_fwd_splitkv_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Nq, Nk, Hq, Hkv, D,
        ctypes.c_float(1.0 / math.sqrt(D)), int(causal), fa.FA_BF16, num_splits, stream)


def _oracle(q, k, v, causal):
    """The oracle's packed form (bottom-right causal), as [B, Nq, Hq, D] and [B, Hq, Nq]."""
    B, Nq, Hq, D = q.shape
    _, Nk, Hkv, _ = k.shape
    o, lse = oracle.attention_varlen(bits(q.reshape(B * Nq, Hq, D)), bits(k.reshape(B * Nk, Hkv, D)),
                                     bits(v.reshape(B * Nk, Hkv, D)), np.arange(B + 1) * Nq, np.arange(B + 1) * Nk,
                                     1 / math.sqrt(D), causal, "bf16")
    return o.reshape(B, Nq, Hq, D), lse.reshape(Hq, B, Nq).transpose(1, 0, 2)


SHAPES = [
    # (B, Nq, Nk, Hq, Hkv, D): paired split-KV (4 query heads per K/V head packed into one tile)
    (1, 4, 6000, 16, 4, 128),
    # unpaired: one query head per K/V head, a single query, ragged last key tile
    (1, 1, 6001, 8, 8, 128),
]


@pytest.mark.parametrize("shape", SHAPES, ids=["paired", "unpaired"])
@pytest.mark.parametrize("causal", [True, False])
def test_noalloc_matches_oracle_twice(shape, causal):
    B, Nq, Nk, Hq, Hkv, D = shape
    n, need = fa.splitkv_plan(B, Nq, Nk, Hq, D, Hkv=Hkv)
    assert n > 1 and 0 < need <= fa.NOALLOC_SCRATCH_BYTES
    for call, seed in enumerate((101, 202)):  # two calls in a row: the scratch keeps the previous contents
        q, k, v = _inputs(seed + Nq, B, Nq, Nk, Hq, Hkv, D)
        qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
        o = torch.full_like(qd, float("nan"))
        lse = torch.full((B, Hq, Nq), float("nan"), device=DEV)
        assert _noalloc_abi(qd, kd, vd, o, lse, causal) == fa.FA_OK
        assert fa.status_sync() == fa.FA_OK
        o_ref, lse_ref = _oracle(q, k, v, causal)
        m = metrics(o.cpu().double().numpy(), lse.cpu().double().numpy(), o_ref, lse_ref)
        assert passes(m), (call, m)
        # and the workspace entry point on the same inputs agrees
        o_ws, lse_ws = fa.fwd_splitkv(qd, kd, vd, causal=causal)
        m2 = metrics(o.cpu().double().numpy(), lse.cpu().double().numpy(), o_ws.cpu().double().numpy(),
                     lse_ws.cpu().double().numpy())
        assert passes(m2), (call, m2)


def test_noalloc_falls_back_to_a_range_count_that_fits():
    """With num_splits = 0 the plan's range count needs more partial-result
    memory than the scratch holds; the call uses the largest count that fits."""
    B, Nq, Nk, Hq, Hkv, D = 1, 16, 65536, 32, 4, 128
    n, need = fa.splitkv_plan(B, Nq, Nk, Hq, D, Hkv=Hkv)
    assert need > fa.NOALLOC_SCRATCH_BYTES  # the automatic count does not fit
    q, k, v = _inputs(7, B, Nq, Nk, Hq, Hkv, D)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o = torch.full_like(qd, float("nan"))
    lse = torch.full((B, Hq, Nq), float("nan"), device=DEV)
    assert _noalloc_abi(qd, kd, vd, o, lse, True) == fa.FA_OK
    assert fa.status_sync() == fa.FA_OK
    o_ref, lse_ref = _oracle(q, k, v, True)
    m = metrics(o.cpu().double().numpy(), lse.cpu().double().numpy(), o_ref, lse_ref)
    assert passes(m), m


def test_noalloc_call_leaves_free_memory_unchanged():
    B, Nq, Nk, Hq, Hkv, D = SHAPES[0]
    q, k, v = (t.to(DEV) for t in _inputs(5, B, Nq, Nk, Hq, Hkv, D))
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), device=DEV)
    assert _noalloc_abi(q, k, v, o, lse, True) == fa.FA_OK  # warm-up: the scratch address is looked up
    assert fa.status_sync() == fa.FA_OK
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert _noalloc_abi(q, k, v, o, lse, False) == fa.FA_OK
    assert fa.status_sync() == fa.FA_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_noalloc_rejects_sizes_beyond_the_scratch():
    # 64 ranges x 256 query rows x 64 heads x (128 + 1) fp32 values is about 540 MB of partial results
    B, Nq, Nk, Hq, D = 1, 256, 65536, 64, 128
    n, need = fa.splitkv_plan(B, Nq, Nk, Hq, D, 64)
    assert need > fa.NOALLOC_SCRATCH_BYTES
    q = torch.zeros(B, Nq, Hq, D, dtype=torch.bfloat16, device=DEV)
    k = torch.zeros(B, 128, Hq, D, dtype=torch.bfloat16, device=DEV)  # never read: the call is refused first
    o = torch.full_like(q, 3.0)
    lse = torch.full((B, Hq, Nq), 3.0, device=DEV)
    stream = torch.cuda.current_stream().cuda_stream
    st = fa.load_library().fa_fwd_splitkv_noalloc(q.data_ptr(), k.data_ptr(), k.data_ptr(), o.data_ptr(),
                                                   lse.data_ptr(), B, Nq, Nk, Hq, Hq, D, ctypes.c_float(0.1), 0,
                                                   fa.FA_BF16, 64, stream)
    assert st == fa.FA_ERR_UNSUPPORTED
    assert "scratch" in fa.last_error()
    torch.cuda.synchronize()
    assert bool((o == 3.0).all()) and bool((lse == 3.0).all())
