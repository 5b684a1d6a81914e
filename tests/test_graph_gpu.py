"""The C-ABI calls captured in a CUDA graph (torch.cuda.graph) and replayed.

bench.py times the forward by replaying a graph of one step, and a caller may
capture the calls the same way: every entry point only enqueues work on the
stream it is given (tensor maps are built on the host, no device memory is
allocated, no synchronisation happens unless the debug switch is set). Each
test warms the entry point up eagerly, captures it with preallocated outputs,
replays the graph on new inputs copied into the captured buffers, and requires
the bits of an eager call on the same inputs.
"""

import pytest
import torch

import exact_attention_151_b200 as fa

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _rand(shape, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(dtype).to(DEV)


def _same(a, b):
    return torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8))


@pytest.mark.parametrize("causal", [False, True])
def test_forward_replayed_matches_eager(causal):
    B, N, H, D = 2, 1000, 4, 128
    q, k, v = (_rand((B, N, H, D), s) for s in (1, 2, 3))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=DEV)
    fa.fwd_into(q, k, v, o, lse, causal=causal)  # warm-up: per-device setup outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fa.fwd_into(q, k, v, o, lse, causal=causal)
    for seed in (11, 12):  # new inputs into the captured buffers
        q.copy_(_rand((B, N, H, D), seed))
        k.copy_(_rand((B, N, H, D), seed + 100))
        g.replay()
        torch.cuda.synchronize()
        assert fa.status_sync() == fa.FA_OK
        o_e, lse_e = fa.fwd(q, k, v, causal=causal)
        torch.cuda.synchronize()
        assert _same(o, o_e) and _same(lse, lse_e)


def test_splitkv_decode_replayed_matches_eager():
    """Two launches per call (the split kernel and the merge kernel)."""
    B, Nq, Nk, Hq, Hkv, D = 2, 1, 6000, 32, 8, 128
    q, k, v = _rand((B, Nq, Hq, D), 4), _rand((B, Nk, Hkv, D), 5), _rand((B, Nk, Hkv, D), 6)
    n, need = fa.splitkv_plan(B, Nq, Nk, Hq, D, Hkv=Hkv)
    assert n > 1
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=DEV)
    fa.fwd_splitkv(q, k, v, causal=True, workspace=ws, o=o, lse=lse)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fa.fwd_splitkv(q, k, v, causal=True, workspace=ws, o=o, lse=lse)
    q.copy_(_rand((B, Nq, Hq, D), 7))
    g.replay()
    torch.cuda.synchronize()
    assert fa.status_sync() == fa.FA_OK
    o_e, lse_e = fa.fwd_splitkv(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert _same(o, o_e) and _same(lse, lse_e)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_replayed_matches_eager(causal):
    """Three launches per call (preprocess, dQ, dK/dV; the persistent kernels
    reset their work-item counters through the preprocess on every replay)."""
    B, N, Hq, Hkv, D = 2, 700, 8, 2, 128
    q, do = _rand((B, N, Hq, D), 8), _rand((B, N, Hq, D), 9)
    k, v = _rand((B, N, Hkv, D), 10), _rand((B, N, Hkv, D), 11)
    o, lse = fa.fwd(q, k, v, causal=causal)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(k)
    ws = torch.empty(fa.bwd_workspace_size(B, N, Hq), dtype=torch.uint8, device=DEV)
    fa.bwd(q, k, v, o, lse, do, causal=causal, dq=dq, dk=dk, dv=dv, workspace=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fa.bwd(q, k, v, o, lse, do, causal=causal, dq=dq, dk=dk, dv=dv, workspace=ws)
    for seed in (21, 22):
        do.copy_(_rand((B, N, Hq, D), seed))
        g.replay()
        torch.cuda.synchronize()
        assert fa.status_sync() == fa.FA_OK
        ref = fa.bwd(q, k, v, o, lse, do, causal=causal)
        torch.cuda.synchronize()
        for x, y in zip((dq, dk, dv), ref):
            assert _same(x, y)
