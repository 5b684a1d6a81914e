"""GPU parity of the sm_100a backward (dQ, dK, dV through the C ABI) against
the fp64 oracle's backward of the definition.

The GPU path is used as a caller would: its own forward gives O and LSE, then
the backward. The oracle recomputes everything in fp64 from the same 16-bit
q, k, v and dO. Small shapes are compared element by element; the published
Llama-7B shape is compared on whole (batch, head) slices, which the oracle
computes independently (heads and batches do not interact).
"""

import numpy as np
import pytest
import torch

import exact_attention_151_b200 as fa
import oracle
from exact_attention_151_b200.inputs import WORKLOADS, Workload, bits, make_dout, make_qkv
from tests.parity import grad_metrics, grad_passes

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _gpu_grads(q, k, v, dout, scale, causal):
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, dout))
    o, lse = fa.fwd(qd, kd, vd, scale=scale, causal=causal)
    # NaN-filled outputs: every element must be overwritten.
    dq, dk, dv = (torch.full_like(qd, float("nan")) for _ in range(3))
    fa.bwd(qd, kd, vd, o, lse, dod, scale=scale, causal=causal, dq=dq, dk=dk, dv=dv)
    assert fa.status_sync() == fa.FA_OK
    return [t.cpu().to(torch.float64).numpy() for t in (dq, dk, dv)]


def _check(w: Workload):
    q, k, v = make_qkv(w)
    dout = make_dout(w)
    got = _gpu_grads(q, k, v, dout, w.softmax_scale, w.causal)
    ref = oracle.attention_backward(bits(q), bits(k), bits(v), bits(dout), w.softmax_scale, w.causal, w.dtype)
    m = grad_metrics(got, ref)
    print(w.name, w.dtype, "causal" if w.causal else "full", m)
    assert grad_passes(m, w.dtype), (w, m)
    return m


EDGE_N = [1, 17, 128, 129, 255, 300]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("N", EDGE_N)
def test_edge_lengths_full_oracle(N, D, dtype, causal):
    _check(Workload(f"bwd_edge_n{N}_d{D}", B=2, N=N, H=2, D=D, dtype=dtype, causal=causal, seed=3 * N + D))


@pytest.mark.parametrize("causal", [False, True])
def test_several_tiles_ragged_tail(causal):
    _check(Workload("bwd_b1h3n1000d128", B=1, N=1000, H=3, D=128, causal=causal, seed=11))


def test_hot_logits_fp16():
    """Large logits (Q ~ N(0, 4^2)), uniform V: the stress distribution."""
    _check(Workload("bwd_hot_b1h2n700d64_fp16", B=1, N=700, H=2, D=64, dtype="fp16", causal=True, q_std=4.0,
                    v_dist="uniform", seed=5))


@pytest.mark.parametrize("name", ["llama7b_b4h32n2048d128_causal", "small_b1h2n256d64"])
def test_published_shape_sampled_heads(name):
    """Full-size call; the oracle checks whole (b, h) slices: first, last and one middle head."""
    w = WORKLOADS[name]
    q, k, v = make_qkv(w)
    dout = make_dout(w)
    got = _gpu_grads(q, k, v, dout, w.softmax_scale, w.causal)
    picks = sorted({(0, 0), (w.B - 1, w.H - 1), (w.B // 2, w.H // 2)})
    for b, h in picks:
        sl = (slice(b, b + 1), slice(None), slice(h, h + 1))
        ref = oracle.attention_backward(bits(q[sl]), bits(k[sl]), bits(v[sl]), bits(dout[sl]), w.softmax_scale,
                                        w.causal, w.dtype)
        m = grad_metrics([g[sl] for g in got], ref)
        print(name, (b, h), m)
        assert grad_passes(m, w.dtype), (name, b, h, m)


def test_deterministic_and_zero_gradient():
    w = Workload("bwd_det", B=2, N=384, H=2, D=128, causal=True, seed=9)
    q, k, v = (t.to(DEV) for t in make_qkv(w))
    dout = make_dout(w).to(DEV)
    o, lse = fa.fwd(q, k, v, causal=True)
    a = fa.bwd(q, k, v, o, lse, dout, causal=True)
    b = fa.bwd(q, k, v, o, lse, dout, causal=True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)  # bitwise: no atomics, fixed order
    z = fa.bwd(q, k, v, o, lse, torch.zeros_like(dout), causal=True)
    assert fa.status_sync() == fa.FA_OK
    for g in z:
        assert not g.any()  # dO = 0 gives exactly 0 (every term has a factor of dO)
