"""GPU parity of the fused sm_100a forward against the fp64 oracle (through the C ABI).

Small shapes are compared element by element with the whole-matrix oracle;
the published configurations at full size are compared on sampled rows that
the oracle computes one by one (every head, first/last rows, both sides of
every 128-row tile boundary, random rows).
"""

import math

import numpy as np
import pytest
import torch

import exact_attention_151_b200 as fa
import oracle
from exact_attention_151_b200.inputs import WORKLOADS, Workload, bits, make_qkv
from tests.parity import metrics, passes, sample_rows

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _run(q, k, v, scale, causal):
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    B, N, H, D = q.shape
    # NaN-filled outputs: every element must be overwritten.
    o = torch.full_like(qd, float("nan"))
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=DEV)
    fa.fwd_into(qd, kd, vd, o, lse, scale=scale, causal=causal)
    assert fa.status_sync() == fa.FA_OK
    return o.cpu().to(torch.float64).numpy(), lse.cpu().to(torch.float64).numpy()


def _check_full(w: Workload, seed=None):
    q, k, v = make_qkv(w, seed)
    o, lse = _run(q, k, v, w.softmax_scale, w.causal)
    o_ref, lse_ref = oracle.attention(bits(q), bits(k), bits(v), w.softmax_scale, w.causal, w.dtype)
    m = metrics(o, lse, o_ref, lse_ref)
    assert passes(m), (w, m)
    return m


EDGE_N = [1, 2, 15, 16, 17, 127, 128, 129, 255, 256, 257, 1000]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("N", EDGE_N)
def test_edge_lengths_full_oracle(N, D, dtype, causal):
    w = Workload(f"edge_n{N}", B=2, N=N, H=2, D=D, dtype=dtype, causal=causal, seed=N + D)
    _check_full(w)


def test_small_config_full_oracle():
    _check_full(WORKLOADS["small_b1h2n256d64"])


def test_small_config_matches_golden_rows():
    """The committed oracle rows for the small configuration (tests/golden)."""
    import json
    import os

    doc = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "small_b1h2n256d64_rows.json")))
    w = WORKLOADS[doc["workload"]]
    q, k, v = make_qkv(w)
    o, lse = _run(q, k, v, w.softmax_scale, w.causal)
    rows = np.array(doc["rows"])
    o_ref = np.array([[float.fromhex(x) for x in r] for r in doc["o"]])
    lse_ref = np.array([float.fromhex(x) for x in doc["lse"]])
    m = metrics(o[rows[:, 0], rows[:, 2], rows[:, 1]], lse[rows[:, 0], rows[:, 1], rows[:, 2]], o_ref, lse_ref)
    assert passes(m), m


def _check_sampled(w: Workload, per_head_random: int = 64, ends: int = 256):
    """Every (b, h) of a published configuration at full size: its first and
    last `ends` rows, the rows on both sides of every 128-row tile boundary,
    and `per_head_random` random rows, each computed one by one by the oracle
    (exact per row); the whole output is checked to be written and finite."""
    q, k, v = make_qkv(w)
    o, lse = _run(q, k, v, w.softmax_scale, w.causal)
    rows = sample_rows(w.B, w.H, w.N, per_head_random, seed=1, ends=ends)
    assert len({(b, h) for b, h, _ in rows.tolist()}) == w.B * w.H
    o_ref, lse_ref = oracle.attention_rows(bits(q), bits(k), bits(v), w.softmax_scale, w.causal, w.dtype, rows)
    m = metrics(o[rows[:, 0], rows[:, 2], rows[:, 1]], lse[rows[:, 0], rows[:, 1], rows[:, 2]], o_ref, lse_ref)
    assert passes(m), (w.name, m)
    # properties at any size: every output written and finite
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    return m


@pytest.mark.parametrize("name", [
    "llama7b_b4h32n2048d128_causal",
    "long_b1h32n8192d128_noncausal",
    "long_b1h32n8192d128_causal",
    "stress_b2h16n4093d64_fp16_causal",
    "stress_hot_b2h16n4093d64_fp16_causal",
    "sweep_n1024_noncausal",
    "sweep_n1024_causal",
    "sweep_n4096_noncausal",
    "sweep_n4096_causal",
    "sweep_n16384_noncausal",
    "sweep_n16384_causal",
    "sweep_n32768_noncausal",
    "sweep_n32768_causal",
])
def test_published_configs_sampled_rows(name):
    _check_sampled(WORKLOADS[name])


def test_stress_logits_really_large():
    """The hot stress variant drives |logit| near 100: LSE must reflect it."""
    w = WORKLOADS["stress_hot_b2h16n4093d64_fp16_causal"]
    q, k, v = make_qkv(w)
    _, lse = _run(q, k, v, w.softmax_scale, w.causal)
    assert np.abs(lse).max() > 60


def test_deterministic_bitwise():
    w = WORKLOADS["llama7b_b4h32n2048d128_causal"].with_(B=1, H=8)
    q, k, v = (t.to(DEV) for t in make_qkv(w))
    o1, l1 = fa.fwd(q, k, v, causal=True)
    o2, l2 = fa.fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1.view(torch.int32), l2.view(torch.int32))


@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_gives_prefix_means(causal):
    """Q = 0: O row i is the mean of the visible V rows, LSE = ln(#visible)."""
    B, N, H, D = 1, 300, 2, 128
    g = torch.Generator().manual_seed(7)
    q = torch.zeros(B, N, H, D, dtype=torch.bfloat16)
    k = torch.randn(B, N, H, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, N, H, D, generator=g).to(torch.bfloat16)
    o, lse = _run(q, k, v, 0.088, causal)
    vd = v.to(torch.float64).numpy()
    if causal:
        cnt = np.arange(1, N + 1, dtype=np.float64)
        ref = np.cumsum(vd, axis=1) / cnt[None, :, None, None]
        ref_lse = np.broadcast_to(np.log(cnt), (B, H, N))
    else:
        ref = np.broadcast_to(vd.mean(axis=1, keepdims=True), vd.shape)
        ref_lse = np.full((B, H, N), math.log(N))
    m = metrics(o, lse, ref, ref_lse)
    assert passes(m), m


def test_logit_shift_invariance():
    """K' = K + u with everything exactly representable: O unchanged within
    tolerance, LSE shifted by scale * q_i . u."""
    B, N, H, D = 1, 384, 2, 64
    g = torch.Generator().manual_seed(3)
    q = torch.randint(-2, 3, (B, N, H, D), generator=g).to(torch.bfloat16)
    k = torch.randint(-2, 3, (B, N, H, D), generator=g).to(torch.bfloat16)
    v = torch.randn(B, N, H, D, generator=g).to(torch.bfloat16)
    u = torch.randint(-4, 5, (D,), generator=g).to(torch.bfloat16)
    scale = 0.125
    o1, l1 = _run(q, k, v, scale, False)
    o2, l2 = _run(q, (k + u).to(torch.bfloat16), v, scale, False)
    shift = scale * np.einsum("bnhd,d->bhn", q.to(torch.float64).numpy(), u.to(torch.float64).numpy())
    assert np.abs(o1 - o2).max() <= 1e-2
    assert np.abs((l2 - l1) - shift).max() <= 2e-3


def test_power_of_two_rescale_is_bit_identical():
    """(Q * 2^a, scale * 2^-a) produces exactly the same logits, hence the same bits."""
    w = Workload("p2", B=1, N=777, H=4, D=128, seed=21)
    q, k, v = (t.to(DEV) for t in make_qkv(w))
    o1, l1 = fa.fwd(q, k, v, scale=w.softmax_scale)
    o2, l2 = fa.fwd((q * 4).contiguous(), k, v, scale=w.softmax_scale / 4)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1.view(torch.int32), l2.view(torch.int32))


def test_guard_bands_untouched():
    """Writes stay inside O and LSE: sentinel padding on both sides survives."""
    w = Workload("guard", B=2, N=129, H=3, D=64, causal=True, seed=4)
    q, k, v = (t.to(DEV) for t in make_qkv(w))
    pad = 4096
    n_o = q.numel()
    o_buf = torch.full((pad + n_o + pad,), -7.0, dtype=torch.bfloat16, device=DEV)
    l_buf = torch.full((pad + w.B * w.H * w.N + pad,), -9.0, dtype=torch.float32, device=DEV)
    o = o_buf[pad:pad + n_o].view(q.shape)
    lse = l_buf[pad:pad + w.B * w.H * w.N].view(w.B, w.H, w.N)
    fa.fwd_into(q, k, v, o, lse, causal=True)
    assert fa.status_sync() == fa.FA_OK
    assert bool((o_buf[:pad] == -7.0).all()) and bool((o_buf[pad + n_o:] == -7.0).all())
    assert bool((l_buf[:pad] == -9.0).all()) and bool((l_buf[pad + w.B * w.H * w.N:] == -9.0).all())


def test_empty_problem_is_noop():
    q = torch.empty(0, 16, 2, 64, dtype=torch.bfloat16, device=DEV)
    o, lse = fa.fwd(q, q, q)
    assert o.numel() == 0 and lse.numel() == 0


def test_host_errors_do_not_launch():
    w = Workload("err", B=1, N=64, H=1, D=64)
    q, k, v = (t.to(DEV) for t in make_qkv(w))
    o = torch.full_like(q, 3.0)
    lse = torch.full((1, 1, 64), 5.0, device=DEV)
    stream = torch.cuda.current_stream().cuda_stream
    st = fa.fwd_ptr(q.data_ptr() + 2, k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), 1, 64, 1, 64,
                    0.125, False, fa.FA_BF16, stream)
    assert st == fa.FA_ERR_MISALIGNED
    st = fa.fwd_ptr(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), 1, 64, 1, 80,
                    0.125, False, fa.FA_BF16, stream)
    assert st == fa.FA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert bool((o == 3.0).all()) and bool((lse == 5.0).all())


def test_memory_is_linear_in_n():
    """The pages' memory claim (O(N), not O(N^2)): a forward at N = 32768
    (B=1, H=16, D=128) runs while less device memory is free than ONE head's
    N x N fp32 score matrix would take (4 GiB), and the call allocates nothing
    (free device memory is the same before and after it)."""
    w = WORKLOADS["sweep_n32768_noncausal"]
    q, k, v = (t.to(DEV) for t in make_qkv(w))
    o1, o2 = torch.empty_like(q), torch.full_like(q, float("nan"))
    l1 = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=DEV)
    l2 = torch.full_like(l1, float("nan"))
    fa.fwd_into(q, k, v, o1, l1)  # warm-up, and the reference bits
    assert fa.status_sync() == fa.FA_OK
    torch.cuda.synchronize()
    scores_one_head = w.N * w.N * 4
    headroom = 2 << 30
    free, _ = torch.cuda.mem_get_info()
    filler = torch.empty(max(free - headroom, 0), dtype=torch.uint8, device=DEV)
    try:
        torch.cuda.synchronize()
        free_before, _ = torch.cuda.mem_get_info()
        assert free_before < scores_one_head, free_before
        fa.fwd_into(q, k, v, o2, l2)
        assert fa.status_sync() == fa.FA_OK
        torch.cuda.synchronize()
        free_after, _ = torch.cuda.mem_get_info()
        assert free_after == free_before
    finally:
        del filler
        torch.cuda.empty_cache()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1.view(torch.int32), l2.view(torch.int32))
