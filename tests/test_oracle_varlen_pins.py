"""Pins for the oracle's packed-sequence / grouped-query / cross-attention form.

Each check ties attention_varlen to something other than itself: the already
pinned dense oracle (exact equality where the two must coincide), head
repetition for grouped queries, per-sequence independence, torch float64
softmax with an explicit bottom-right mask, and 50-digit brute force.
"""

import math
from decimal import Decimal, getcontext

import numpy as np
import pytest
import torch

import oracle
from exact_attention_151_b200.inputs import bits

rng = np.random.default_rng(99)


def _rand16(shape, dtype="bf16", std=1.0):
    t = (torch.from_numpy(rng.standard_normal(shape).astype(np.float32)) * std)
    t = t.to(torch.bfloat16 if dtype == "bf16" else torch.float16)
    return t, bits(t)


def _cu(lengths):
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)


@pytest.mark.parametrize("causal", [False, True])
def test_equal_lengths_match_dense_oracle_exactly(causal):
    B, N, H, D = 3, 70, 2, 16
    q, Q = _rand16((B, N, H, D))
    k, K = _rand16((B, N, H, D))
    v, V = _rand16((B, N, H, D))
    o, lse = oracle.attention(Q, K, V, 0.25, causal, "bf16")
    ov, lv = oracle.attention_varlen(Q.reshape(B * N, H, D), K.reshape(B * N, H, D), V.reshape(B * N, H, D),
                                     _cu([N] * B), _cu([N] * B), 0.25, causal, "bf16")
    np.testing.assert_array_equal(ov.reshape(B, N, H, D), o)
    np.testing.assert_array_equal(lv.reshape(H, B, N).transpose(1, 0, 2), lse)


@pytest.mark.parametrize("causal", [False, True])
def test_grouped_heads_equal_repeated_heads(causal):
    """Hq = 6 query heads over Hkv = 2 K/V heads: identical to full multi-head
    attention on K/V with each head repeated 3 times."""
    lens_q, lens_k = [5, 40, 17], [9, 40, 33]
    Tq, Tk, Hq, Hkv, D = sum(lens_q), sum(lens_k), 6, 2, 8
    _, Q = _rand16((Tq, Hq, D))
    _, K = _rand16((Tk, Hkv, D))
    _, V = _rand16((Tk, Hkv, D))
    o, lse = oracle.attention_varlen(Q, K, V, _cu(lens_q), _cu(lens_k), 0.3, causal, "bf16")
    Kr, Vr = np.repeat(K, 3, axis=1), np.repeat(V, 3, axis=1)
    o2, lse2 = oracle.attention_varlen(Q, Kr, Vr, _cu(lens_q), _cu(lens_k), 0.3, causal, "bf16")
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)


def test_sequences_are_independent():
    """Packing sequences together changes nothing: each equals its own one-sequence call."""
    lens_q, lens_k = [1, 31, 0, 64], [4, 31, 7, 100]
    Hq, Hkv, D = 4, 2, 16
    _, Q = _rand16((sum(lens_q), Hq, D))
    _, K = _rand16((sum(lens_k), Hkv, D))
    _, V = _rand16((sum(lens_k), Hkv, D))
    cq, ck = _cu(lens_q), _cu(lens_k)
    o, lse = oracle.attention_varlen(Q, K, V, cq, ck, 0.2, True, "bf16")
    for b in range(len(lens_q)):
        qs, ks = slice(cq[b], cq[b + 1]), slice(ck[b], ck[b + 1])
        ob, lb = oracle.attention_varlen(Q[qs], K[ks], V[ks], [0, lens_q[b]], [0, lens_k[b]], 0.2, True, "bf16")
        np.testing.assert_array_equal(o[qs], ob)
        np.testing.assert_array_equal(lse[:, qs], lb)


@pytest.mark.parametrize("nq,nk", [(50, 50), (30, 80), (80, 30), (1, 64), (64, 1)])
@pytest.mark.parametrize("causal", [False, True])
def test_cross_attention_matches_torch_with_bottom_right_mask(nq, nk, causal):
    """torch float64 softmax with the mask j <= i + nk - nq; rows with no
    visible key give O = 0 and LSE = -inf."""
    H, D = 2, 32
    q, Q = _rand16((nq, H, D))
    k, K = _rand16((nk, H, D))
    v, V = _rand16((nk, H, D))
    scale = 1.0 / math.sqrt(D)
    o, lse = oracle.attention_varlen(Q, K, V, [0, nq], [0, nk], scale, causal, "bf16")
    qd, kd, vd = (t.to(torch.float64).permute(1, 0, 2) for t in (q, k, v))
    s = scale * qd @ kd.transpose(-1, -2)
    if causal:
        i = torch.arange(nq)[:, None]
        j = torch.arange(nk)[None, :]
        s = s.masked_fill(j > i + nk - nq, float("-inf"))
    ref_lse = torch.logsumexp(s, dim=-1)
    w = torch.softmax(s, dim=-1).nan_to_num(0.0)  # empty rows: all weights 0
    ref_o = (w @ vd).permute(1, 0, 2).numpy()
    np.testing.assert_allclose(o, ref_o, rtol=0, atol=1e-12)
    finite = np.isfinite(ref_lse.numpy())
    np.testing.assert_allclose(lse[finite], ref_lse.numpy()[finite], rtol=0, atol=1e-12)
    assert np.all(np.isneginf(lse[~finite]))
    if causal and nq > nk:
        assert (~finite).sum() == H * (nq - nk)  # the first nq - nk rows see nothing
        assert np.all(o[: nq - nk] == 0.0)


def test_cross_attention_brute_force():
    getcontext().prec = 50
    nq, nk, D = 3, 5, 2
    qv = rng.integers(-3, 4, size=(nq, 1, D)).astype(np.float32)
    kv = rng.integers(-3, 4, size=(nk, 1, D)).astype(np.float32)
    vv = rng.integers(-5, 6, size=(nk, 1, D)).astype(np.float32)
    Q, K, V = (bits(torch.from_numpy(x).to(torch.float16)) for x in (qv, kv, vv))
    scale = 0.375
    o, lse = oracle.attention_varlen(Q, K, V, [0, nq], [0, nk], scale, True, "fp16")
    for i in range(nq):
        js = [j for j in range(nk) if j <= i + nk - nq]
        s = [Decimal(repr(scale)) * sum(Decimal(int(qv[i, 0, d])) * Decimal(int(kv[j, 0, d])) for d in range(D))
             for j in js]
        w = [x.exp() for x in s]
        tot = sum(w)
        for d in range(D):
            exact = sum(wj * Decimal(int(vv[j, 0, d])) for wj, j in zip(w, js)) / tot
            assert abs(o[i, 0, d] - float(exact)) < 1e-13
        assert abs(lse[0, i] - float(tot.ln())) < 1e-13


def test_bad_segments_rejected():
    _, Q = _rand16((4, 1, 8))
    with pytest.raises(ValueError):
        oracle.attention_varlen(Q, Q, Q, [0, 3, 2, 4], [0, 1, 2, 4], 1.0, False, "bf16")
    with pytest.raises(ValueError):
        oracle.attention_varlen(Q, Q, Q, [0, 5], [0, 4], 1.0, False, "bf16")
