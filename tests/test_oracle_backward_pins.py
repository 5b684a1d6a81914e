"""Pins for the oracle's backward (dQ, dK, dV of sum(O * dO)).

Independent of the oracle's code: central finite differences of a float64
torch forward, torch float64 autograd (the special case that reduces to
library routines), closed forms (dO = 0; uniform attention), and invariants
of the softmax (keys' dK sum to zero; a constant added to V changes nothing
but O).
"""

import numpy as np
import pytest
import torch

import oracle
from exact_attention_151_b200.inputs import Workload, bits, make_qkv


def _torch_forward(q, k, v, scale, causal):
    qd, kd, vd = (t.permute(0, 2, 1, 3) for t in (q, k, v))
    s = scale * qd @ kd.transpose(-1, -2)
    if causal:
        n = s.shape[-1]
        s = s.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), float("-inf"))
    return (torch.softmax(s, dim=-1) @ vd).permute(0, 2, 1, 3)


def _case(N=40, H=2, D=16, causal=True, seed=3, B=2):
    w = Workload("bwd", B=B, N=N, H=H, D=D, causal=causal, seed=seed)
    q, k, v = make_qkv(w)
    g = torch.Generator().manual_seed(seed + 100)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    return w, q, k, v, do


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_float64_autograd(causal):
    w, q, k, v, do = _case(causal=causal)
    dq, dk, dv = oracle.attention_backward(bits(q), bits(k), bits(v), bits(do), w.softmax_scale, causal, "bf16")
    qd, kd, vd = (t.double().requires_grad_() for t in (q, k, v))
    o = _torch_forward(qd, kd, vd, w.softmax_scale, causal)
    (o * do.double()).sum().backward()
    np.testing.assert_allclose(dq, qd.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk, kd.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, vd.grad.numpy(), rtol=0, atol=1e-12)


def test_matches_central_finite_differences():
    """d/dx of sum(O * dO) by (L(x + h) - L(x - h)) / 2h on a few entries of each input."""
    w, q, k, v, do = _case(N=12, H=1, D=8, causal=True, B=1)
    dq, dk, dv = oracle.attention_backward(bits(q), bits(k), bits(v), bits(do), w.softmax_scale, True, "bf16")
    base = [t.double() for t in (q, k, v)]
    dod = do.double()
    rng = np.random.default_rng(0)
    h = 1e-5
    for which, grad in enumerate((dq, dk, dv)):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, s)) for s in base[which].shape)
            plus = [t.clone() for t in base]
            minus = [t.clone() for t in base]
            plus[which][idx] += h
            minus[which][idx] -= h
            lp = (_torch_forward(*plus, w.softmax_scale, True) * dod).sum().item()
            lm = (_torch_forward(*minus, w.softmax_scale, True) * dod).sum().item()
            assert abs((lp - lm) / (2 * h) - grad[idx]) < 1e-7


def test_zero_output_gradient_gives_zero():
    w, q, k, v, do = _case()
    dq, dk, dv = oracle.attention_backward(bits(q), bits(k), bits(v), bits(torch.zeros_like(do)),
                                           w.softmax_scale, True, "bf16")
    assert not dq.any() and not dk.any() and not dv.any()


def test_uniform_attention_value_gradient():
    """Q = 0 gives uniform weights over the visible keys: dV_j = sum_{i >= j} dO_i / (i + 1) (causal)."""
    w, q, k, v, do = _case(N=30, causal=True)
    q = torch.zeros_like(q)
    _, _, dv = oracle.attention_backward(bits(q), bits(k), bits(v), bits(do), w.softmax_scale, True, "bf16")
    dod = do.double().numpy()
    cnt = np.arange(1, w.N + 1, dtype=np.float64)[None, :, None, None]
    weighted = dod / cnt
    ref = np.flip(np.cumsum(np.flip(weighted, axis=1), axis=1), axis=1)  # suffix sums over queries i >= j
    np.testing.assert_allclose(dv, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_key_gradients_sum_to_zero(causal):
    """Each softmax row's dS sums to zero, so sum_j dK_j = 0 for every (b, h)."""
    w, q, k, v, do = _case(causal=causal)
    _, dk, _ = oracle.attention_backward(bits(q), bits(k), bits(v), bits(do), w.softmax_scale, causal, "bf16")
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)


def test_value_shift_leaves_q_and_k_gradients():
    """V + c (one constant vector for all keys) shifts O by c; dQ and dK are unchanged."""
    w, q, k, v, do = _case(causal=True)
    g = torch.Generator().manual_seed(5)
    v = torch.randint(-8, 9, v.shape, generator=g).to(torch.bfloat16)  # integers: v + c stays exact
    c = torch.randint(-3, 4, (w.D,), generator=g).to(torch.bfloat16)
    v2 = (v + c).to(torch.bfloat16)
    assert torch.equal(v2.double(), v.double() + c.double())  # exact in bf16 for these values
    a = oracle.attention_backward(bits(q), bits(k), bits(v), bits(do), w.softmax_scale, True, "bf16")
    b = oracle.attention_backward(bits(q), bits(k), bits(v2), bits(do), w.softmax_scale, True, "bf16")
    np.testing.assert_allclose(b[0], a[0], rtol=0, atol=1e-11)
    np.testing.assert_allclose(b[1], a[1], rtol=0, atol=1e-11)
    np.testing.assert_array_equal(b[2], a[2])
