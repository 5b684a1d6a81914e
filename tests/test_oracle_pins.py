"""Pins for the fp64 CPU oracle, each against something other than itself.

Every check below fixes a fact the mathematics (or a library routine) decides
independently of the oracle's code: closed forms, invariances, exhaustive
comparison with library conversions, arbitrary-precision brute force, and the
handbook's tiled online-softmax routine as a second, differently ordered
statement of the same result. A dropped term, a wrong sign or index, a
transposed operand, a wrong mask or a wrong log base fails at least one.
"""

import math
from decimal import Decimal, getcontext

import numpy as np
import pytest
import torch

import oracle
from exact_attention_151_b200.inputs import Workload, bits, make_qkv

rng = np.random.default_rng(1234)


def _to16(x: np.ndarray, dtype: str) -> np.ndarray:
    """float array -> 16-bit patterns (values must already be representable)."""
    t = torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16 if dtype == "bf16" else torch.float16)
    back = t.to(torch.float64).numpy()
    assert np.array_equal(back, np.asarray(x, dtype=np.float64)), "test input not exactly representable"
    return bits(t)


def _ints(shape, lo, hi):
    return rng.integers(lo, hi + 1, size=shape).astype(np.float64)


# ---------------------------------------------------------------- decoding


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_decode16_exhaustive_matches_library(dtype):
    """Every one of the 65536 patterns widens exactly as torch/numpy do."""
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.decode16(pats, dtype)
    if dtype == "fp16":
        ref = pats.view(np.float16).astype(np.float64)
    else:
        ref = torch.from_numpy(pats.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


# ---------------------------------------------------------------- closed forms


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("mode", ["full", "rows", "tiled"])
def test_zero_query_gives_mean_of_visible_values(causal, dtype, mode):
    """Q = 0 makes every logit 0: O is the mean of the visible V rows
    (a prefix mean when causal) and LSE = ln(#visible)."""
    B, N, H, D = 2, 37, 3, 8
    q = np.zeros((B, N, H, D))
    k = _ints((B, N, H, D), -4, 4)
    v = _ints((B, N, H, D), -8, 8)
    Q, K, V = _to16(q, dtype), _to16(k, dtype), _to16(v, dtype)
    scale = 0.37
    if mode == "full":
        o, lse = oracle.attention(Q, K, V, scale, causal, dtype)
    elif mode == "tiled":
        o, lse = oracle.tiled_reference(Q, K, V, scale, causal, dtype, block_size=16)
    else:
        rows = np.array([(b, h, i) for b in range(B) for h in range(H) for i in range(N)])
        orows, lrows = oracle.attention_rows(Q, K, V, scale, causal, dtype, rows)
        o = np.empty((B, N, H, D))
        lse = np.empty((B, H, N))
        for r, (b, h, i) in enumerate(rows):
            o[b, i, h] = orows[r]
            lse[b, h, i] = lrows[r]
    for b in range(B):
        for h in range(H):
            for i in range(N):
                nvis = i + 1 if causal else N
                expect = v[b, :nvis, h, :].mean(axis=0)
                np.testing.assert_allclose(o[b, i, h], expect, rtol=0, atol=1e-13)
                assert abs(lse[b, h, i] - math.log(nvis)) <= 1e-13


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_single_key_returns_its_value(dtype):
    """N = 1: the only key gets weight 1, so O = V_0 and LSE = scale * q.k_0."""
    B, N, H, D = 3, 1, 2, 16
    q, k, v = _ints((B, N, H, D), -3, 3), _ints((B, N, H, D), -3, 3), _ints((B, N, H, D), -9, 9)
    scale = 0.125
    for causal in (False, True):
        o, lse = oracle.attention(_to16(q, dtype), _to16(k, dtype), _to16(v, dtype), scale, causal, dtype)
        np.testing.assert_array_equal(o, v)
        expect = scale * np.einsum("bnhd,bnhd->bhn", q, k)
        np.testing.assert_array_equal(lse, expect)


def test_hand_worked_two_key_case():
    """q = 1, k = (0, 1), v = (0, 1), scale = 1: logits (0, 1), so the
    non-causal row is e/(1+e) with LSE ln(1+e); causal row 0 sees only key 0."""
    q = np.ones((1, 2, 1, 1))
    k = np.array([0.0, 1.0]).reshape(1, 2, 1, 1)
    v = np.array([0.0, 1.0]).reshape(1, 2, 1, 1)
    Q, K, V = _to16(q, "bf16"), _to16(k, "bf16"), _to16(v, "bf16")
    o, lse = oracle.attention(Q, K, V, 1.0, False, "bf16")
    e = math.e
    assert abs(o[0, 0, 0, 0] - e / (1 + e)) < 1e-15 and abs(o[0, 1, 0, 0] - e / (1 + e)) < 1e-15
    assert abs(lse[0, 0, 0] - math.log(1 + e)) < 1e-15
    o, lse = oracle.attention(Q, K, V, 1.0, True, "bf16")
    assert o[0, 0, 0, 0] == 0.0 and lse[0, 0, 0] == 0.0
    assert abs(o[0, 1, 0, 0] - e / (1 + e)) < 1e-15 and abs(lse[0, 0, 1] - math.log(1 + e)) < 1e-15


@pytest.mark.parametrize("causal", [False, True])
def test_constant_values_are_reproduced(causal):
    """V = c for every key: the weights sum to one, so O = c exactly up to rounding."""
    B, N, H, D = 1, 50, 2, 8
    q = _ints((B, N, H, D), -6, 6)
    k = _ints((B, N, H, D), -6, 6)
    c = _ints((1, 1, 1, D), -5, 5)
    v = np.broadcast_to(c, (B, N, H, D)).copy()
    o, _ = oracle.attention(_to16(q, "bf16"), _to16(k, "bf16"), _to16(v, "bf16"), 0.3, causal, "bf16")
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_row_constant_logit_shift(causal):
    """K' = K + u adds scale*(q_i.u) to every logit of row i: O is unchanged,
    LSE moves by exactly that amount (max subtraction / normalisation)."""
    B, N, H, D = 1, 40, 2, 8
    q = _ints((B, N, H, D), -4, 4)
    k = _ints((B, N, H, D), -4, 4)
    v = _ints((B, N, H, D), -8, 8)
    u = _ints((1, 1, 1, D), -20, 20)
    scale = 0.25
    o1, l1 = oracle.attention(_to16(q, "bf16"), _to16(k, "bf16"), _to16(v, "bf16"), scale, causal, "bf16")
    o2, l2 = oracle.attention(_to16(q, "bf16"), _to16(k + u, "bf16"), _to16(v, "bf16"), scale, causal, "bf16")
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-11)
    shift = scale * np.einsum("bnhd,d->bhn", q, u.reshape(D))
    np.testing.assert_allclose(l2 - l1, shift, rtol=0, atol=1e-10)


def test_permutation_properties():
    """Non-causal: permuting K and V rows together leaves O unchanged;
    permuting Q rows permutes O rows (rows are independent)."""
    B, N, H, D = 1, 64, 2, 16
    q, k, v = _ints((B, N, H, D), -3, 3), _ints((B, N, H, D), -3, 3), _ints((B, N, H, D), -7, 7)
    scale = 0.2
    f = lambda a: _to16(a, "bf16")
    o, lse = oracle.attention(f(q), f(k), f(v), scale, False, "bf16")
    perm = rng.permutation(N)
    o_kv, lse_kv = oracle.attention(f(q), f(k[:, perm]), f(v[:, perm]), scale, False, "bf16")
    np.testing.assert_allclose(o_kv, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse_kv, lse, rtol=0, atol=1e-12)
    o_q, lse_q = oracle.attention(f(q[:, perm]), f(k), f(v), scale, False, "bf16")
    np.testing.assert_array_equal(o_q, o[:, perm])
    np.testing.assert_array_equal(lse_q, lse[:, :, perm])


def test_causal_row_sees_exactly_its_prefix():
    """Causal row i equals the non-causal result on the first i+1 keys only."""
    B, N, H, D = 1, 33, 1, 8
    q, k, v = _ints((B, N, H, D), -3, 3), _ints((B, N, H, D), -3, 3), _ints((B, N, H, D), -7, 7)
    f = lambda a: _to16(a, "bf16")
    o, lse = oracle.attention(f(q), f(k), f(v), 0.3, True, "bf16")
    for i in [0, 1, 5, 17, 32]:
        # a single query row against a prefix: the query position does not matter without a mask
        o_pref, l_pref = oracle.attention(f(np.repeat(q[:, i:i + 1], i + 1, axis=1)), f(k[:, :i + 1]),
                                          f(v[:, :i + 1]), 0.3, False, "bf16")
        np.testing.assert_array_equal(o[0, i, 0], o_pref[0, 0, 0])
        assert lse[0, 0, i] == l_pref[0, 0, 0]


# ---------------------------------------------------------------- brute force


def _decimal_attention(q, k, v, scale, causal):
    """Arbitrary-precision (50 digits) softmax-weighted sum, straight from the formula."""
    getcontext().prec = 50
    B, N, H, D = q.shape
    o = np.empty((B, N, H, D))
    lse = np.empty((B, H, N))
    sc = Decimal(repr(scale))
    for b in range(B):
        for h in range(H):
            for i in range(N):
                js = range(i + 1) if causal else range(N)
                s = [sc * sum(Decimal(repr(float(q[b, i, h, d]))) * Decimal(repr(float(k[b, j, h, d]))) for d in range(D))
                     for j in js]
                w = [x.exp() for x in s]
                tot = sum(w)
                for d in range(D):
                    o[b, i, h, d] = float(sum(wj * Decimal(repr(float(v[b, j, h, d]))) for wj, j in zip(w, js)) / tot)
                lse[b, h, i] = float(tot.ln())
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 1, 1, 1), (1, 3, 1, 2), (2, 5, 2, 3), (1, 8, 1, 4)])
def test_brute_force_tiny_shapes(shape, causal):
    q, k, v = _ints(shape, -5, 5), _ints(shape, -5, 5), _ints(shape, -9, 9)
    scale = 0.4375  # exactly representable, so Decimal(repr()) is the true value
    o, lse = oracle.attention(_to16(q, "fp16"), _to16(k, "fp16"), _to16(v, "fp16"), scale, causal, "fp16")
    o_ref, lse_ref = _decimal_attention(q, k, v, scale, causal)
    np.testing.assert_allclose(o, o_ref, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-14, atol=1e-13)


# ---------------------------------------------------------------- second statement


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,block", [(1, 128), (2, 1), (7, 3), (16, 16), (100, 7), (129, 128), (300, 64), (257, 32)])
def test_tiled_routine_matches_definition(N, block, causal):
    """The handbook's tiled online softmax (normalising at every block) reaches
    the same O and LSE as the materialised definition, to fp64 rounding."""
    w = Workload("pin", B=1, N=N, H=2, D=16, causal=causal, seed=N * 7 + block)
    q, k, v = make_qkv(w)
    Q, K, V = bits(q), bits(k), bits(v)
    o, lse = oracle.attention(Q, K, V, w.softmax_scale, causal, "bf16")
    o_t, lse_t = oracle.tiled_reference(Q, K, V, w.softmax_scale, causal, "bf16", block_size=block)
    np.testing.assert_allclose(o_t, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse_t, lse, rtol=0, atol=1e-12)


def test_large_logits_stay_finite_and_match_tiled():
    """Logits near 100 (the stress regime): no overflow, both statements agree."""
    w = Workload("hot", B=1, N=300, H=1, D=64, dtype="fp16", causal=True, q_std=16.0, v_dist="uniform", seed=3)
    q, k, v = make_qkv(w)
    Q, K, V = bits(q), bits(k), bits(v)
    o, lse = oracle.attention(Q, K, V, w.softmax_scale, True, "fp16")
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    assert np.abs(lse).max() > 30  # the regime is really exercised
    o_t, lse_t = oracle.tiled_reference(Q, K, V, w.softmax_scale, True, "fp16", block_size=64)
    np.testing.assert_allclose(o_t, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse_t, lse, rtol=0, atol=1e-11)


# ---------------------------------------------------------------- library routine


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_float64_softmax(causal):
    """The special case that reduces to library routines: torch.softmax on
    float64 scores (with a -inf mask above the diagonal), then a matmul."""
    w = Workload("lib", B=2, N=200, H=3, D=64, causal=causal, seed=11)
    q, k, v = make_qkv(w)
    o, lse = oracle.attention(bits(q), bits(k), bits(v), w.softmax_scale, causal, "bf16")
    qd, kd, vd = (t.to(torch.float64).permute(0, 2, 1, 3) for t in (q, k, v))
    s = w.softmax_scale * qd @ kd.transpose(-1, -2)
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(w.N, w.N, dtype=torch.bool), 1), float("-inf"))
    ref_o = (torch.softmax(s, dim=-1) @ vd).permute(0, 2, 1, 3).numpy()
    ref_lse = torch.logsumexp(s, dim=-1).numpy()
    np.testing.assert_allclose(o, ref_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- internal consistency


@pytest.mark.parametrize("causal", [False, True])
def test_rows_mode_is_bit_identical_to_full(causal):
    w = Workload("rows", B=2, N=130, H=2, D=64, causal=causal, seed=5)
    q, k, v = make_qkv(w)
    Q, K, V = bits(q), bits(k), bits(v)
    o, lse = oracle.attention(Q, K, V, w.softmax_scale, causal, "bf16")
    rows = np.array([(b, h, i) for b in range(2) for h in range(2) for i in (0, 1, 63, 64, 127, 128, 129)])
    orow, lrow = oracle.attention_rows(Q, K, V, w.softmax_scale, causal, "bf16", rows)
    for r, (b, h, i) in enumerate(rows):
        np.testing.assert_array_equal(orow[r], o[b, i, h])
        assert lrow[r] == lse[b, h, i]


def test_thread_count_does_not_change_results():
    w = Workload("thr", B=1, N=90, H=2, D=32, causal=True, seed=9)
    q, k, v = make_qkv(w)
    a = oracle.attention(bits(q), bits(k), bits(v), w.softmax_scale, True, "bf16", nthreads=1)
    b = oracle.attention(bits(q), bits(k), bits(v), w.softmax_scale, True, "bf16", nthreads=5)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_bad_arguments_are_rejected():
    z = np.zeros((1, 2, 1, 4), dtype=np.uint16)
    with pytest.raises(TypeError):
        oracle.attention(z.astype(np.float32), z, z, 1.0, False, "bf16")
    with pytest.raises(ValueError):
        oracle.attention_rows(z, z, z, 1.0, False, "bf16", [(0, 0, 5)])


def test_golden_rows_unchanged():
    """Regression: the committed oracle rows for the small configuration
    (written by tests/golden/make_golden.py from the oracle) still reproduce."""
    import json
    import os

    from exact_attention_151_b200.inputs import WORKLOADS

    path = os.path.join(os.path.dirname(__file__), "golden", "small_b1h2n256d64_rows.json")
    doc = json.load(open(path))
    w = WORKLOADS[doc["workload"]]
    q, k, v = make_qkv(w)
    o, lse = oracle.attention_rows(bits(q), bits(k), bits(v), w.softmax_scale, w.causal, w.dtype, doc["rows"])
    np.testing.assert_array_equal(o, np.array([[float.fromhex(x) for x in r] for r in doc["o"]]))
    np.testing.assert_array_equal(lse, np.array([float.fromhex(x) for x in doc["lse"]]))
