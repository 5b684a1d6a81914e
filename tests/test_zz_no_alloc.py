"""The split-KV entry point that allocates nothing (fa_fwd_splitkv_noalloc).

Some callers must not allocate device memory on the call path (their GPU
memory is reserved up front by another allocator, or they cannot handle an
out-of-memory failure mid-request); this entry point keeps its partial
results in a scratch buffer compiled into the library instead of a caller
workspace. The test calls it through the C ABI twice in a row and compares
each result with the workspace entry point fa_fwd_splitkv on the same inputs,
within the parity tolerance used throughout the tests. It sits in its own
file, collected last, and depends on no other test.
"""

import ctypes
import math

import pytest
import torch

import exact_attention_151_b200 as fa
from tests.parity import metrics, passes

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _inputs(seed, B=1, Nq=4, Nk=6000, Hq=16, Hkv=4, D=128):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Nq, Hq, D, generator=g).to(torch.bfloat16).to(DEV)
    k = torch.randn(B, Nk, Hkv, D, generator=g).to(torch.bfloat16).to(DEV)
    v = torch.randn(B, Nk, Hkv, D, generator=g).to(torch.bfloat16).to(DEV)
    return q, k, v


def _noalloc_abi(q, k, v, o, lse, causal, num_splits=0):
    B, Nq, Hq, D = q.shape
    _, Nk, Hkv, _ = k.shape
    stream = torch.cuda.current_stream().cuda_stream
    return fa.load_library().fa_fwd_splitkv_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Nq, Nk, Hq, Hkv, D,
        ctypes.c_float(1.0 / math.sqrt(D)), int(causal), fa.FA_BF16, num_splits, stream)


@pytest.mark.parametrize("causal", [True, False])
def test_noalloc_matches_workspace_entry_point_twice(causal):
    for call, seed in enumerate((101, 202)):  # two calls in a row: the scratch keeps the previous contents
        q, k, v = _inputs(seed)
        n, need = fa.splitkv_plan(q.shape[0], q.shape[1], k.shape[1], q.shape[2], q.shape[3], Hkv=k.shape[2])
        assert n > 1 and 0 < need <= fa.NOALLOC_SCRATCH_BYTES
        o_ref, lse_ref = fa.fwd_splitkv(q, k, v, causal=causal)
        o = torch.full_like(q, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        assert _noalloc_abi(q, k, v, o, lse, causal) == fa.FA_OK
        assert fa.status_sync() == fa.FA_OK
        m = metrics(o.cpu().double().numpy(), lse.cpu().double().numpy(), o_ref.cpu().double().numpy(),
                    lse_ref.cpu().double().numpy())
        assert passes(m), (call, m)


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
