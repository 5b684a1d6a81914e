"""Pins for the oracle's backward in the general form (attention_backward_varlen):
packed sequences, grouped-query heads, queries and keys of different lengths
with the causal mask aligned at the bottom-right corner.

Independent of the oracle's code: torch float64 autograd through an explicit
masked softmax with the K/V heads repeated for their query heads (the special
case that reduces to library routines), central finite differences of a
float64 torch forward, and identities: with equal lengths and one query head
per K/V head it is the (separately pinned) dense backward; grouped heads give
the sum of the repeated heads' dense gradients; sequences are independent;
rows and keys with nothing visible get zero gradients; each K/V head's dK sums
to zero over the keys.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_attention_151_b200.inputs import bits


def _rand(shape, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(torch.bfloat16)


def _torch_grads(q, k, v, do, nq, nk, scale, causal):
    """One sequence: q, do [nq, Hq, D]; k, v [nk, Hkv, D] (bf16). float64 autograd
    through softmax(scale Q K^T + bottom-right mask) V with K/V heads repeated."""
    Hq, Hkv = q.shape[1], k.shape[1]
    G = Hq // Hkv
    qd, kd, vd = (t.double().requires_grad_() for t in (q, k, v))
    kr = kd.repeat_interleave(G, dim=1).permute(1, 0, 2)  # [Hq, nk, D]
    vr = vd.repeat_interleave(G, dim=1).permute(1, 0, 2)
    s = scale * qd.permute(1, 0, 2) @ kr.transpose(-1, -2)  # [Hq, nq, nk]
    if causal:
        i = torch.arange(nq)[:, None]
        j = torch.arange(nk)[None, :]
        s = s.masked_fill(j > i + (nk - nq), float("-inf"))
    p = torch.softmax(s, dim=-1)
    p = torch.nan_to_num(p, nan=0.0)  # rows with no visible key: weight 0
    o = (p @ vr).permute(1, 0, 2)
    (o * do.double()).sum().backward()
    zero = lambda t, like: t if t is not None else torch.zeros_like(like)  # noqa: E731
    return zero(qd.grad, qd).numpy(), zero(kd.grad, kd).numpy(), zero(vd.grad, vd).numpy()


def _packed(lens_q, lens_k, Hq, Hkv, D, seed):
    tq, tk = sum(lens_q), sum(lens_k)
    q = _rand((tq, Hq, D), seed)
    k = _rand((tk, Hkv, D), seed + 1)
    v = _rand((tk, Hkv, D), seed + 2)
    do = _rand((tq, Hq, D), seed + 3)
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int64)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int64)
    return q, k, v, do, cu_q, cu_k


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2), (3, 1)])
def test_matches_torch_float64_autograd(causal, Hq, Hkv):
    lens_q, lens_k = [7, 20, 13, 1, 9], [19, 6, 13, 5, 0]  # cross lengths, a key-less sequence
    D = 16
    q, k, v, do, cu_q, cu_k = _packed(lens_q, lens_k, Hq, Hkv, D, seed=Hq * 10 + Hkv)
    scale = 1 / math.sqrt(D)
    dq, dk, dv = oracle.attention_backward_varlen(bits(q), bits(k), bits(v), bits(do), cu_q, cu_k, scale, causal,
                                                  "bf16")
    for b in range(len(lens_q)):
        a, e = cu_q[b], cu_q[b + 1]
        ka, ke = cu_k[b], cu_k[b + 1]
        rq, rk, rv = _torch_grads(q[a:e], k[ka:ke], v[ka:ke], do[a:e], e - a, ke - ka, scale, causal)
        np.testing.assert_allclose(dq[a:e], rq, rtol=0, atol=1e-12)
        np.testing.assert_allclose(dk[ka:ke], rk, rtol=0, atol=1e-12)
        np.testing.assert_allclose(dv[ka:ke], rv, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_equal_lengths_one_head_per_kv_is_the_dense_backward(causal):
    B, N, H, D = 2, 33, 3, 16
    q, k, v, do = (_rand((B, N, H, D), s) for s in (41, 42, 43, 44))
    scale = 0.2
    dense = oracle.attention_backward(bits(q), bits(k), bits(v), bits(do), scale, causal, "bf16")
    cu = np.arange(B + 1) * N
    packed = oracle.attention_backward_varlen(bits(q.reshape(B * N, H, D)), bits(k.reshape(B * N, H, D)),
                                              bits(v.reshape(B * N, H, D)), bits(do.reshape(B * N, H, D)), cu, cu,
                                              scale, causal, "bf16")
    for a, b in zip(dense, packed):
        np.testing.assert_array_equal(a.reshape(B * N, H, D), b)


@pytest.mark.parametrize("causal", [False, True])
def test_grouped_heads_sum_the_repeated_heads_gradients(causal):
    """Hq = 4 query heads over Hkv = 2 K/V heads equals multi-head attention on
    K/V repeated per query head, with dK, dV of a K/V head the sum over its
    repeats (to rounding: the sums are associated differently)."""
    N, Hq, Hkv, D = 29, 4, 2, 16
    G = Hq // Hkv
    q, do = _rand((1, N, Hq, D), 51), _rand((1, N, Hq, D), 54)
    k, v = _rand((1, N, Hkv, D), 52), _rand((1, N, Hkv, D), 53)
    kr, vr = k.repeat_interleave(G, dim=2), v.repeat_interleave(G, dim=2)
    scale = 0.25
    dq_r, dk_r, dv_r = oracle.attention_backward(bits(q), bits(kr), bits(vr), bits(do), scale, causal, "bf16")
    cu = np.array([0, N])
    dq, dk, dv = oracle.attention_backward_varlen(bits(q[0]), bits(k[0]), bits(v[0]), bits(do[0]), cu, cu, scale,
                                                  causal, "bf16")
    np.testing.assert_array_equal(dq, dq_r[0])
    np.testing.assert_allclose(dk, dk_r[0].reshape(N, Hkv, G, D).sum(axis=2), rtol=0, atol=1e-13)
    np.testing.assert_allclose(dv, dv_r[0].reshape(N, Hkv, G, D).sum(axis=2), rtol=0, atol=1e-13)


def test_sequences_are_independent():
    lens_q, lens_k = [12, 5, 30], [8, 17, 30]
    q, k, v, do, cu_q, cu_k = _packed(lens_q, lens_k, 4, 2, 16, seed=61)
    full = oracle.attention_backward_varlen(bits(q), bits(k), bits(v), bits(do), cu_q, cu_k, 0.3, True, "bf16")
    for b in range(3):
        a, e, ka, ke = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        one = oracle.attention_backward_varlen(bits(q[a:e]), bits(k[ka:ke]), bits(v[ka:ke]), bits(do[a:e]),
                                               [0, e - a], [0, ke - ka], 0.3, True, "bf16")
        np.testing.assert_array_equal(full[0][a:e], one[0])
        np.testing.assert_array_equal(full[1][ka:ke], one[1])
        np.testing.assert_array_equal(full[2][ka:ke], one[2])


def test_nothing_visible_gives_zero_gradients():
    """nq > nk, causal: the first nq - nk queries see no key (dQ = 0); with
    nq < nk, causal: keys past ... are all seen; a key-less sequence has no dK."""
    lens_q, lens_k = [10, 3], [4, 9]
    q, k, v, do, cu_q, cu_k = _packed(lens_q, lens_k, 2, 1, 16, seed=71)
    dq, dk, dv = oracle.attention_backward_varlen(bits(q), bits(k), bits(v), bits(do), cu_q, cu_k, 0.3, True, "bf16")
    assert np.all(dq[:6] == 0.0)            # queries 0..5 of sequence 0 see no key (i + 4 - 10 < 0)
    assert np.any(dq[6:10] != 0.0)
    # sequence 1: 3 queries over 9 keys, query i sees keys j <= i + 6: every key is seen by the last query
    assert np.all(np.any(dv[4:] != 0.0, axis=(1, 2)))


def test_dk_sums_to_zero_over_keys():
    """Each softmax row's dS sums to zero, so for every (sequence, K/V head)
    sum_j dK_j = scale sum_i (sum_j dS_ij) Q_i = 0."""
    lens_q, lens_k = [15, 40], [33, 40]
    q, k, v, do, cu_q, cu_k = _packed(lens_q, lens_k, 6, 2, 16, seed=81)
    _, dk, _ = oracle.attention_backward_varlen(bits(q), bits(k), bits(v), bits(do), cu_q, cu_k, 0.25, True, "bf16")
    for b in range(2):
        tot = dk[cu_k[b]:cu_k[b + 1]].sum(axis=0)
        assert np.abs(tot).max() < 1e-12


def test_matches_central_finite_differences():
    """d/dx of sum(O * dO) by (L(x + h) - L(x - h)) / 2h for sampled entries,
    on a cross-length causal sequence with grouped heads."""
    nq, nk, Hq, Hkv, D = 6, 9, 2, 1, 8
    q, k, v, do, cu_q, cu_k = _packed([nq], [nk], Hq, Hkv, D, seed=91)
    scale = 0.35
    grads = oracle.attention_backward_varlen(bits(q), bits(k), bits(v), bits(do), cu_q, cu_k, scale, True, "bf16")

    def loss(qq, kk, vv):
        kr = kk.repeat_interleave(Hq // Hkv, dim=1).permute(1, 0, 2)
        vr = vv.repeat_interleave(Hq // Hkv, dim=1).permute(1, 0, 2)
        s = scale * qq.permute(1, 0, 2) @ kr.transpose(-1, -2)
        i = torch.arange(nq)[:, None]
        j = torch.arange(nk)[None, :]
        s = s.masked_fill(j > i + (nk - nq), float("-inf"))
        o = (torch.softmax(s, dim=-1) @ vr).permute(1, 0, 2)
        return float((o * do.double()).sum())

    base = [t.double() for t in (q, k, v)]
    rng = np.random.default_rng(3)
    h = 1e-5
    for which, grad in enumerate(grads):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, s)) for s in base[which].shape)
            plus = [t.clone() for t in base]
            minus = [t.clone() for t in base]
            plus[which][idx] += h
            minus[which][idx] -= h
            fd = (loss(*plus) - loss(*minus)) / (2 * h)
            assert abs(fd - grad[idx]) < 1e-7, (which, idx, fd, grad[idx])
