"""GPU parity of the backward's general form (fa_bwd_gqa through the C ABI):
grouped-query heads (a K/V head's gradient sums over the query heads that
read it), queries and keys of different lengths with the causal mask aligned
at the bottom-right corner, against the fp64 oracle's backward of the packed
form. The GPU forward supplies O and LSE, as a caller's would."""

import math

import numpy as np
import pytest
import torch

import exact_attention_151_b200 as fa
import oracle
from exact_attention_151_b200.inputs import bits
from tests.parity import grad_metrics, grad_passes

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _randn(shape, seed, dtype):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(dtype)


def _run(B, Nq, Nk, Hq, Hkv, D, dtype, causal, seed):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    q = _randn((B, Nq, Hq, D), seed, tdt)
    k = _randn((B, Nk, Hkv, D), seed + 1, tdt)
    v = _randn((B, Nk, Hkv, D), seed + 2, tdt)
    do = _randn((B, Nq, Hq, D), seed + 3, tdt)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o, lse = fa.fwd(qd, kd, vd, causal=causal)
    # NaN-filled outputs: every element must be overwritten
    dq = torch.full_like(qd, float("nan"))
    dk = torch.full_like(kd, float("nan"))
    dv = torch.full_like(kd, float("nan"))
    fa.bwd(qd, kd, vd, o, lse, dod, causal=causal, dq=dq, dk=dk, dv=dv)
    assert fa.status_sync() == fa.FA_OK
    got = [t.cpu().to(torch.float64).numpy() for t in (dq, dk, dv)]
    ref = oracle.attention_backward_varlen(bits(q.reshape(B * Nq, Hq, D)), bits(k.reshape(B * Nk, Hkv, D)),
                                           bits(v.reshape(B * Nk, Hkv, D)), bits(do.reshape(B * Nq, Hq, D)),
                                           np.arange(B + 1) * Nq, np.arange(B + 1) * Nk, 1 / math.sqrt(D), causal,
                                           dtype)
    ref = [ref[0].reshape(B, Nq, Hq, D), ref[1].reshape(B, Nk, Hkv, D), ref[2].reshape(B, Nk, Hkv, D)]
    return got, ref


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(256, 256), (300, 300), (128, 1000), (1000, 128), (513, 700), (700, 513),
                                   (1, 300), (300, 1)])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (4, 1)])
def test_gqa_cross_lengths(Nq, Nk, Hq, Hkv, causal):
    got, ref = _run(2, Nq, Nk, Hq, Hkv, 128, "bf16", causal, seed=Nq * 7 + Nk + Hq * 3 + Hkv)
    m = grad_metrics(got, ref)
    assert grad_passes(m, "bf16"), m


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_gqa_d64(dtype, causal):
    got, ref = _run(1, 777, 640, 6, 2, 64, dtype, causal, seed=5)
    m = grad_metrics(got, ref)
    assert grad_passes(m, dtype), m


def test_rows_and_keys_with_nothing_visible():
    """Causal with Nq > Nk: the first Nq - Nk queries see no key (dQ = 0,
    exactly); every key is seen by some query."""
    B, Nq, Nk, Hq, Hkv, D = 1, 700, 200, 4, 2, 128
    got, ref = _run(B, Nq, Nk, Hq, Hkv, D, "bf16", True, seed=17)
    assert np.all(got[0][:, : Nq - Nk] == 0.0)
    m = grad_metrics(got, ref)
    assert grad_passes(m, "bf16"), m


@pytest.mark.parametrize("Nq,Nk", [(0, 300), (300, 0)])
def test_empty_side_gives_zero_gradients(Nq, Nk):
    """No queries: dK = dV = 0; no keys: dQ = 0 (O = 0, LSE = -inf from the forward)."""
    B, Hq, Hkv, D = 2, 4, 2, 64
    q = torch.randn(B, Nq, Hq, D, device=DEV).to(torch.bfloat16)
    k = torch.randn(B, Nk, Hkv, D, device=DEV).to(torch.bfloat16)
    v = torch.randn(B, Nk, Hkv, D, device=DEV).to(torch.bfloat16)
    do = torch.randn(B, Nq, Hq, D, device=DEV).to(torch.bfloat16)
    o, lse = fa.fwd(q, k, v, causal=True) if Nq > 0 else (torch.empty_like(q), torch.empty(B, Hq, 0, device=DEV))
    dq = torch.full_like(q, float("nan"))
    dk = torch.full_like(k, float("nan"))
    dv = torch.full_like(k, float("nan"))
    fa.bwd(q, k, v, o, lse, do, causal=True, dq=dq, dk=dk, dv=dv)
    assert fa.status_sync() == fa.FA_OK
    for t in (dq, dk, dv):
        assert bool((t == 0).all())


def test_gqa_deterministic_bitwise():
    B, Nq, Nk, Hq, Hkv, D = 1, 1000, 1200, 8, 2, 128
    g = torch.Generator().manual_seed(3)
    q, do = (torch.randn(B, Nq, Hq, D, generator=g).to(torch.bfloat16).to(DEV) for _ in range(2))
    k, v = (torch.randn(B, Nk, Hkv, D, generator=g).to(torch.bfloat16).to(DEV) for _ in range(2))
    o, lse = fa.fwd(q, k, v, causal=True)
    a = fa.bwd(q, k, v, o, lse, do, causal=True)
    b = fa.bwd(q, k, v, o, lse, do, causal=True)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))


def test_llama_shape_with_grouped_heads_sampled_slices():
    """Llama-2/Mistral-style grouped heads at the Llama-7B size: B=4, N=2048,
    32 query heads over 8 K/V heads, causal; the oracle on two whole batches'
    worth of one K/V group each (batches and groups do not interact)."""
    B, N, Hq, Hkv, D = 4, 2048, 32, 8, 128
    G = Hq // Hkv
    g = torch.Generator().manual_seed(29)
    q = torch.randn(B, N, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(B, N, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, N, Hkv, D, generator=g).to(torch.bfloat16)
    do = torch.randn(B, N, Hq, D, generator=g).to(torch.bfloat16)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o, lse = fa.fwd(qd, kd, vd, causal=True)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, lse, dod, causal=True)
    assert fa.status_sync() == fa.FA_OK
    dq, dk, dv = (t.cpu().to(torch.float64).numpy() for t in (dq, dk, dv))
    assert np.isfinite(dq).all() and np.isfinite(dk).all() and np.isfinite(dv).all()
    for b, hk in ((0, 0), (3, 5)):
        hs = slice(hk * G, (hk + 1) * G)
        cu = np.array([0, N])
        ref = oracle.attention_backward_varlen(bits(q[b, :, hs]), bits(k[b, :, hk:hk + 1]), bits(v[b, :, hk:hk + 1]),
                                               bits(do[b, :, hs]), cu, cu, 1 / math.sqrt(D), True, "bf16")
        m = grad_metrics([dq[b, :, hs], dk[b, :, hk:hk + 1], dv[b, :, hk:hk + 1]], ref)
        assert grad_passes(m, "bf16"), (b, hk, m)


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("fp16", 64)])
@pytest.mark.parametrize("causal", [False, True])
def test_packed_sequences(dtype, D, causal):
    """fa_bwd_varlen on sequences of different lengths (including an empty
    one and one without keys) against the oracle's packed backward."""
    lens_q = [1, 0, 257, 128, 700, 33, 300, 5]
    lens_k = [5, 3, 257, 300, 700, 1, 100, 0]
    Hq, Hkv = 8, 2
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    q = _randn((sum(lens_q), Hq, D), 11, tdt)
    k = _randn((sum(lens_k), Hkv, D), 12, tdt)
    v = _randn((sum(lens_k), Hkv, D), 13, tdt)
    do = _randn((sum(lens_q), Hq, D), 14, tdt)
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    cq, ck = torch.from_numpy(cu_q).to(DEV), torch.from_numpy(cu_k).to(DEV)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o, lse = fa.fwd_varlen(qd, kd, vd, cq, ck, max(lens_q), causal=causal)
    dq = torch.full_like(qd, float("nan"))
    dk = torch.full_like(kd, float("nan"))
    dv = torch.full_like(kd, float("nan"))
    fa.bwd_varlen(qd, kd, vd, o, lse, dod, cq, ck, max(lens_q), max(lens_k), causal=causal, dq=dq, dk=dk, dv=dv)
    assert fa.status_sync() == fa.FA_OK
    got = [t.cpu().to(torch.float64).numpy() for t in (dq, dk, dv)]
    ref = oracle.attention_backward_varlen(bits(q), bits(k), bits(v), bits(do), cu_q, cu_k, 1 / math.sqrt(D), causal,
                                           dtype)
    m = grad_metrics(got, ref)
    assert grad_passes(m, dtype), m


def test_packed_equals_dense_bitwise():
    """Equal-length packed sequences give exactly the dense call's bits."""
    B, N, Hq, Hkv, D = 3, 300, 4, 2, 128
    g = torch.Generator().manual_seed(23)
    q, do = (torch.randn(B, N, Hq, D, generator=g).to(torch.bfloat16).to(DEV) for _ in range(2))
    k, v = (torch.randn(B, N, Hkv, D, generator=g).to(torch.bfloat16).to(DEV) for _ in range(2))
    o, lse = fa.fwd(q, k, v, causal=True)
    a = fa.bwd(q, k, v, o, lse, do, causal=True)
    cu = torch.arange(B + 1, dtype=torch.int32, device=DEV) * N
    lse_p = lse.permute(1, 0, 2).reshape(Hq, B * N).contiguous()
    b = fa.bwd_varlen(q.reshape(B * N, Hq, D), k.reshape(B * N, Hkv, D), v.reshape(B * N, Hkv, D),
                      o.reshape(B * N, Hq, D), lse_p, do.reshape(B * N, Hq, D), cu, cu, N, N, causal=True)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x.reshape(y.shape).view(torch.int16), y.view(torch.int16))


def test_packed_inconsistent_offsets_are_reported():
    H, D = 2, 64
    q = torch.randn(100, H, D, device=DEV).to(torch.bfloat16)
    cu_q = torch.tensor([0, 60, 40, 100], dtype=torch.int32, device=DEV)  # decreasing: sequence 1 is invalid
    cu_k = torch.tensor([0, 30, 60, 100], dtype=torch.int32, device=DEV)
    o = torch.zeros_like(q)
    lse = torch.zeros(H, 100, device=DEV)
    fa.bwd_varlen(q, q, q, o, lse, q, cu_q, cu_k, 60, 40, causal=False)
    assert fa.status_sync() == fa.FA_ERR_INVALID_ARG
    assert fa.status_sync() == fa.FA_OK


def test_gradients_at_16_byte_offsets_match_aligned_bitwise():
    """Gradient buffers that are only 16-byte aligned take the 16-byte store
    path of the epilogues (32-byte aligned ones the 32-byte path); both write
    the same bits."""
    B, N, Hq, Hkv, D = 2, 300, 4, 2, 128
    g = torch.Generator().manual_seed(41)
    q, do = (torch.randn(B, N, Hq, D, generator=g).to(torch.bfloat16).to(DEV) for _ in range(2))
    k, v = (torch.randn(B, N, Hkv, D, generator=g).to(torch.bfloat16).to(DEV) for _ in range(2))
    o, lse = fa.fwd(q, k, v, causal=True)
    a = fa.bwd(q, k, v, o, lse, do, causal=True)

    def offset_like(t):  # a view 16 bytes past a 256-byte aligned allocation
        buf = torch.full((t.numel() + 8,), float("nan"), dtype=t.dtype, device=DEV)
        view = buf[8:].view(t.shape)
        assert view.data_ptr() % 32 == 16
        return view

    dq, dk, dv = offset_like(q), offset_like(k), offset_like(k)
    fa.bwd(q, k, v, o, lse, do, causal=True, dq=dq, dk=dk, dv=dv)
    assert fa.status_sync() == fa.FA_OK
    for x, y in zip(a, (dq, dk, dv)):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))
