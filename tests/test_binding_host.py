"""The Python binding's argument marshalling, on the CPU.

The binding only checks arguments and passes pointers and sizes to the C ABI.
Here the CUDA-only pieces around it are replaced: the library by a recorder
that answers the host-only queries (range plan, workspace size) from the real
library and records every compute call, torch's stream and device context by
stand-ins, and the device check by one that accepts CPU tensors. Each entry
point then runs end to end on CPU tensors, which checks both the arguments it
hands to the C ABI (sizes, dtype code, scale, mask, workspace size) and that
wrong shapes, dtypes or devices are refused before any call is made (the C ABI
only sees raw pointers, so a mis-sized output would be written out of bounds).
"""

import contextlib
import ctypes
import math

import pytest
import torch

import exact_attention_151_b200 as fa


class _Recorder:
    """Stands in for the loaded library: compute entry points are recorded and
    return FA_OK; the host-only queries go to the real library."""

    def __init__(self, real):
        self.real = real
        self.calls = []

    def __getattr__(self, name):
        if name in ("fa_fwd_splitkv_plan", "fa_bwd_workspace_size", "fa_status_string", "fa_last_error"):
            return getattr(self.real, name)

        def call(*args):
            self.calls.append((name, args))
            return fa.FA_OK

        return call


@pytest.fixture
def rec(monkeypatch):
    r = _Recorder(fa.load_library())
    monkeypatch.setattr(fa, "load_library", lambda: r)

    def check_cpu(device=None, **tensors):
        for name, t in tensors.items():
            if not t.is_contiguous():
                raise ValueError(f"{name} must be contiguous")
            if device is not None and t.device != device:
                raise ValueError(f"{name} is on {t.device}")

    monkeypatch.setattr(fa, "_check_cuda", check_cpu)

    class _Stream:
        cuda_stream = 1234

    monkeypatch.setattr(torch.cuda, "current_stream", lambda device=None: _Stream())
    monkeypatch.setattr(torch.cuda, "device", lambda device=None: contextlib.nullcontext())
    return r


def _t(shape, dtype=torch.bfloat16):
    return torch.zeros(shape, dtype=dtype)


def _val(x):
    return x.value if isinstance(x, (ctypes.c_float, ctypes.c_int, ctypes.c_size_t)) else x


def test_fwd_dense_and_grouped(rec):
    q, k = _t((2, 100, 4, 64)), _t((2, 100, 4, 64))
    o, lse = fa.fwd(q, k, k, causal=True)
    assert o.shape == q.shape and lse.shape == (2, 4, 100) and lse.dtype == torch.float32
    name, args = rec.calls[-1]
    assert name == "fa_fwd"
    assert [_val(a) for a in args[5:]] == [2, 100, 4, 64, pytest.approx(1 / 8), 1, fa.FA_BF16, 1234]
    kg = _t((2, 300, 2, 64), torch.float16)
    fa.fwd(q.half(), kg, kg, scale=0.5)
    name, args = rec.calls[-1]
    assert name == "fa_fwd_gqa"
    assert [_val(a) for a in args[5:]] == [2, 100, 300, 4, 2, 64, 0.5, 0, fa.FA_FP16, 1234]


def test_fwd_rejects_bad_arguments_before_any_call(rec):
    q = _t((2, 100, 4, 64))
    with pytest.raises(ValueError):
        fa.fwd_into(q, q, q, _t((2, 100, 4, 32)), _t((2, 4, 100), torch.float32))      # o of the wrong shape
    with pytest.raises(ValueError):
        fa.fwd_into(q, q, q, torch.empty_like(q), _t((2, 100, 4), torch.float32))     # lse transposed
    with pytest.raises(TypeError):
        fa.fwd_into(q, q.half(), q, torch.empty_like(q), _t((2, 4, 100), torch.float32))
    with pytest.raises(TypeError):
        fa.fwd(q.float(), q.float(), q.float())
    with pytest.raises(ValueError):
        fa.fwd_into(q, q, q, torch.empty_like(q), _t((2, 100, 4), torch.float32).transpose(1, 2))  # not contiguous
    assert rec.calls == []


def test_fwd_varlen(rec):
    q, k = _t((150, 4, 128)), _t((90, 2, 128))
    cu_q = torch.tensor([0, 100, 150], dtype=torch.int32)
    cu_k = torch.tensor([0, 40, 90], dtype=torch.int32)
    o, lse = fa.fwd_varlen(q, k, k, cu_q, cu_k, 100, causal=True)
    assert o.shape == q.shape and lse.shape == (4, 150)
    name, args = rec.calls[-1]
    assert name == "fa_fwd_varlen"
    assert [_val(a) for a in args[7:]] == [2, 100, 150, 90, 4, 2, 128, pytest.approx(1 / math.sqrt(128)), 1,
                                           fa.FA_BF16, 1234]
    n = len(rec.calls)
    with pytest.raises(ValueError):
        fa.fwd_varlen(q, k, k, cu_q, cu_k, 100, lse=_t((150, 4), torch.float32))      # lse must be [Hq, total_q]
    with pytest.raises(ValueError):
        fa.fwd_varlen(q, k, k, cu_q, cu_k, 100, o=_t((150, 4, 64)))
    with pytest.raises(ValueError):
        fa.fwd_varlen(q, k, k, cu_q, cu_k, 100, o=_t((150, 4, 128), torch.float16))   # o dtype differs from q
    with pytest.raises(TypeError):
        fa.fwd_varlen(q, k, k, cu_q.long(), cu_k, 100)
    assert len(rec.calls) == n


def test_fwd_splitkv(rec):
    q, k = _t((8, 1, 32, 128)), _t((8, 8192, 8, 128))
    o, lse = fa.fwd_splitkv(q, k, k, causal=True)
    name, args = rec.calls[-1]
    assert name == "fa_fwd_splitkv"
    n_splits, need = fa.splitkv_plan(8, 1, 8192, 32, 128, Hkv=8)
    assert [_val(a) for a in args[5:14]] == [8, 1, 8192, 32, 8, 128, pytest.approx(1 / math.sqrt(128)), 1,
                                            fa.FA_BF16]
    assert args[14] == 0 and args[16] == max(need, 1) and args[17] == 1234
    n = len(rec.calls)
    with pytest.raises(ValueError):
        fa.fwd_splitkv(q, k, k, o=_t((8, 1, 32, 64)))
    with pytest.raises(ValueError):
        fa.fwd_splitkv(q, k, k, lse=_t((8, 1, 32), torch.float32))
    with pytest.raises(TypeError):
        fa.fwd_splitkv(q, k, k, workspace=torch.zeros(need, dtype=torch.float32))
    with pytest.raises(ValueError):
        fa.fwd_splitkv(q, _t((4, 8192, 8, 128)), _t((4, 8192, 8, 128)))               # batch differs
    with pytest.raises(TypeError):
        fa.fwd_splitkv(q, k, k.half())
    assert len(rec.calls) == n


def test_fwd_splitkv_noalloc(rec):
    q, k = _t((1, 4, 16, 128)), _t((1, 6000, 4, 128))
    o, lse = torch.empty_like(q), _t((1, 16, 4), torch.float32)
    fa.fwd_splitkv_noalloc(q, k, k, o, lse, causal=True)
    name, args = rec.calls[-1]
    assert name == "fa_fwd_splitkv_noalloc"
    assert [_val(a) for a in args[5:]] == [1, 4, 6000, 16, 4, 128, pytest.approx(1 / math.sqrt(128)), 1, fa.FA_BF16,
                                           0, 1234]
    n = len(rec.calls)
    with pytest.raises(ValueError):
        fa.fwd_splitkv_noalloc(q, k, k, o, _t((1, 4, 16), torch.float32))
    with pytest.raises(ValueError):
        fa.fwd_splitkv_noalloc(q, k, k, o.half(), lse)
    with pytest.raises(TypeError):
        fa.fwd_splitkv_noalloc(q, k.half(), k.half(), o, lse)
    assert len(rec.calls) == n


def test_bwd_dense_grouped_and_packed(rec):
    q, k = _t((2, 100, 4, 64)), _t((2, 100, 4, 64))
    lse = _t((2, 4, 100), torch.float32)
    dq, dk, dv = fa.bwd(q, k, k, q, lse, q, causal=True)
    assert dq.shape == q.shape and dk.shape == k.shape and dv.shape == k.shape
    name, args = rec.calls[-1]
    assert name == "fa_bwd"
    ws = fa.bwd_workspace_size(2, 100, 4)
    assert [_val(a) for a in args[9:]][:8] == [2, 100, 4, 64, pytest.approx(1 / 8), 1, fa.FA_BF16, args[16]]
    assert args[17] == ws and args[18] == 1234
    kg = _t((2, 300, 2, 64))
    fa.bwd(q, kg, kg, q, lse, q)
    assert rec.calls[-1][0] == "fa_bwd_gqa"
    qp, kp = _t((150, 4, 128)), _t((90, 2, 128))
    cu_q = torch.tensor([0, 100, 150], dtype=torch.int32)
    cu_k = torch.tensor([0, 40, 90], dtype=torch.int32)
    lp = _t((4, 150), torch.float32)
    fa.bwd_varlen(qp, kp, kp, qp, lp, qp, cu_q, cu_k, 100, 50, causal=True)
    name, args = rec.calls[-1]
    assert name == "fa_bwd_varlen"
    assert [_val(a) for a in args[11:19]] == [2, 100, 50, 150, 90, 4, 2, 128]
    n = len(rec.calls)
    with pytest.raises(ValueError):
        fa.bwd_varlen(qp, kp, kp, qp, lp, qp, cu_q, cu_k, 100, 50, dk=_t((90, 4, 128)))   # dk shaped like q
    with pytest.raises(ValueError):
        fa.bwd_varlen(qp, kp, kp, qp, lp, qp, cu_q, cu_k, 100, 50, dq=_t((150, 4, 128), torch.float16))
    with pytest.raises(TypeError):
        fa.bwd_varlen(qp, kp, kp, qp, lp, qp, cu_q, cu_k, 100, 50, workspace=torch.zeros(64, dtype=torch.int32))
    with pytest.raises(ValueError):
        fa.bwd(q, k, k, q, lse, q, dv=_t((2, 100, 4, 32)))
    with pytest.raises(ValueError):
        fa.bwd(q, k, k, q, _t((2, 100, 4), torch.float32), q)
    assert len(rec.calls) == n


def test_host_tensors_are_refused_before_any_call():
    """The real device check: pointers from host memory never reach the library."""
    q = _t((1, 8, 2, 64))
    with pytest.raises(ValueError, match="CUDA tensor"):
        fa.fwd(q, q, q)
    with pytest.raises(ValueError, match="CUDA tensor"):
        fa.fwd_splitkv_noalloc(q, q, q, torch.empty_like(q), _t((1, 2, 8), torch.float32))
