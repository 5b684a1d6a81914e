"""B200-native exact attention: O = softmax(scale * Q K^T [+ causal]) V with per-row LSE, and its gradients.

Thin Python binding over the C ABI in ``include/fa.h`` (library
``libfa_b200.so``, built in-tree for sm_100a). This module only marshals
arguments (pointers, sizes, the current CUDA stream); every step of the
computation runs in the library's CUDA kernel. There is no fallback: if the
library is missing or the device is not an sm_100 GPU, calls raise.

Tensors use the [B, N, H, D] layout (contiguous, bf16 or fp16, D in {64, 128});
LSE is float32 [B, H, N] in natural-log units of the scaled logits.
"""

from __future__ import annotations

import ctypes
import math
import os

__all__ = ["fwd", "fwd_into", "fwd_varlen", "fwd_splitkv", "splitkv_plan", "fwd_ptr", "bwd", "bwd_varlen",
           "bwd_workspace_size", "status_sync", "FaError", "library_path", "load_library",
           "FA_OK", "FA_ERR_INVALID_ARG", "FA_ERR_UNSUPPORTED", "FA_ERR_MISALIGNED", "FA_ERR_CUDA",
           "FA_ERR_TIMEOUT", "FA_ERR_DEVICE_CHECK", "EXPORTED_SYMBOLS", "load_checking_library"]

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_MISALIGNED = 3
FA_ERR_CUDA = 4
FA_ERR_TIMEOUT = 5
FA_ERR_DEVICE_CHECK = 6

FA_BF16 = 0
FA_FP16 = 1

# Every entry point declared in include/fa.h.
EXPORTED_SYMBOLS = ("fa_status_string", "fa_last_error", "fa_fwd", "fa_fwd_gqa", "fa_fwd_varlen",
                    "fa_fwd_splitkv", "fa_fwd_splitkv_plan", "fa_fwd_splitkv_noalloc", "fa_status_sync",
                    "fa_fwd_debug", "fa_bwd", "fa_bwd_gqa", "fa_bwd_varlen", "fa_bwd_workspace_size")

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_FILE = os.path.join(_HERE, "libfa_b200.so")
_CHECKS_LIB_FILE = os.path.join(_HERE, "libfa_b200_checks.so")
_lib = None
_checks_lib = None


class FaError(RuntimeError):
    """A non-OK status from the C library."""

    def __init__(self, code: int, where: str):
        self.code = code
        detail = last_error() if code == FA_ERR_CUDA else ""
        super().__init__(f"{where}: {status_string(code)} (code {code})" + (f" [{detail}]" if detail else ""))


def library_path() -> str:
    return _LIB_FILE


def load_library():
    """Load the in-tree CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        _lib = _open(_LIB_FILE)
    return _lib


def load_checking_library():
    """Load the checking build (libfa_b200_checks.so: device-side index checks
    before every global store, reported as FA_ERR_DEVICE_CHECK); same C ABI."""
    global _checks_lib
    if _checks_lib is None:
        _checks_lib = _open(_CHECKS_LIB_FILE)
    return _checks_lib


def _open(path):
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library {path} is missing; build it with "
                           "`python -m exact_attention_151_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.fa_status_string.argtypes = [i32]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_last_error.argtypes = []
    lib.fa_last_error.restype = ctypes.c_char_p
    fwd_args = [vp, vp, vp, vp, vp, i64, i64, i64, i64, ctypes.c_float, i32, i32, vp]
    lib.fa_fwd.argtypes = fwd_args
    lib.fa_fwd.restype = i32
    lib.fa_fwd_debug.argtypes = fwd_args + [ctypes.c_uint64, i32]
    lib.fa_fwd_debug.restype = i32
    lib.fa_fwd_gqa.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, ctypes.c_float, i32, i32, vp]
    lib.fa_fwd_gqa.restype = i32
    lib.fa_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, ctypes.c_float, i32,
                                  i32, vp]
    lib.fa_fwd_varlen.restype = i32
    lib.fa_fwd_splitkv.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, ctypes.c_float, i32, i32, i32, vp,
                                   ctypes.c_size_t, vp]
    lib.fa_fwd_splitkv.restype = i32
    lib.fa_fwd_splitkv_plan.argtypes = [i64, i64, i64, i64, i64, i64, i32, ctypes.POINTER(i32),
                                        ctypes.POINTER(ctypes.c_size_t)]
    lib.fa_fwd_splitkv_plan.restype = i32
    lib.fa_fwd_splitkv_noalloc.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, ctypes.c_float, i32, i32,
                                           i32, vp]
    lib.fa_fwd_splitkv_noalloc.restype = i32
    lib.fa_bwd_workspace_size.argtypes = [i64, i64, i64, ctypes.POINTER(ctypes.c_size_t)]
    lib.fa_bwd_workspace_size.restype = i32
    lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, ctypes.c_float, i32, i32, vp,
                           ctypes.c_size_t, vp]
    lib.fa_bwd.restype = i32
    lib.fa_bwd_gqa.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, ctypes.c_float, i32,
                               i32, vp, ctypes.c_size_t, vp]
    lib.fa_bwd_gqa.restype = i32
    lib.fa_bwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, i64,
                                  ctypes.c_float, i32, i32, vp, ctypes.c_size_t, vp]
    lib.fa_bwd_varlen.restype = i32
    lib.fa_status_sync.argtypes = [vp]
    lib.fa_status_sync.restype = i32
    return lib


def last_error() -> str:
    """Detail of the last FA_ERR_CUDA on this thread ("" if none)."""
    return load_library().fa_last_error().decode()


def status_string(code: int) -> str:
    return load_library().fa_status_string(int(code)).decode()


def fwd_ptr(q: int, k: int, v: int, o: int, lse: int, B: int, N: int, H: int, D: int, scale: float,
            causal: bool, dtype: int, stream: int, *, wait_limit_ns: int | None = None,
            withhold_v_load: bool = False) -> int:
    """Raw C-ABI call with integer device pointers; returns the fa_status code."""
    lib = load_library()
    if wait_limit_ns is None and not withhold_v_load:
        return lib.fa_fwd(q, k, v, o, lse, B, N, H, D, ctypes.c_float(scale), int(bool(causal)), int(dtype),
                          stream)
    return lib.fa_fwd_debug(q, k, v, o, lse, B, N, H, D, ctypes.c_float(scale), int(bool(causal)), int(dtype),
                            stream, int(wait_limit_ns or 0), int(bool(withhold_v_load)))


def status_sync(stream: int | None = None) -> int:
    """Synchronise the stream, then read and clear the device status word."""
    import torch

    s = torch.cuda.current_stream().cuda_stream if stream is None else stream
    return load_library().fa_status_sync(s)


def _dtype_code(t) -> int:
    import torch

    if t.dtype == torch.bfloat16:
        return FA_BF16
    if t.dtype == torch.float16:
        return FA_FP16
    raise TypeError(f"q/k/v must be bfloat16 or float16, got {t.dtype}")


def _check_cuda(device=None, **tensors):
    """Every tensor is a contiguous CUDA tensor, on ``device`` when given (the
    library receives raw pointers: a host pointer or another GPU's memory
    would reach the kernels unchecked)."""
    for name, t in tensors.items():
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if device is not None and t.device != device:
            raise ValueError(f"{name} is on {t.device}; every tensor must be on {device}")


def _check_like(name, t, shape, dtype):
    """A caller-provided output has exactly the shape and dtype the kernels write."""
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype} {list(shape)}, got {t.dtype} {list(t.shape)}")


def _check_qkv4(q, k, v):
    """q [B, Nq, Hq, D] and k, v [B, Nk, Hkv, D] of one 16-bit dtype."""
    if q.dim() != 4 or k.dim() != 4 or v.shape != k.shape:
        raise ValueError("q must be [B, Nq, Hq, D] and k, v [B, Nk, Hkv, D]")
    if k.shape[0] != q.shape[0] or k.shape[3] != q.shape[3]:
        raise ValueError("q and k/v disagree on batch or head dimension")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k and v must share one dtype")
    _dtype_code(q)


def fwd_into(q, k, v, o, lse, scale: float | None = None, causal: bool = False, **debug) -> None:
    """Forward into caller-provided ``o`` ([B,Nq,Hq,D]) and ``lse`` (fp32 [B,Hq,Nq]).

    k and v may have their own length Nk and Hkv heads (Hq % Hkv == 0); with
    causal=True the mask is aligned at the bottom-right corner.
    """
    import torch

    if q.dim() != 4 or k.dim() != 4 or v.shape != k.shape or o.shape != q.shape:
        raise ValueError("q, o must be [B, Nq, Hq, D] and k, v [B, Nk, Hkv, D]")
    B, Nq, Hq, D = q.shape
    Bk, Nk, Hkv, Dk = k.shape
    if Bk != B or Dk != D:
        raise ValueError("q and k/v disagree on batch or head dimension")
    if tuple(lse.shape) != (B, Hq, Nq) or lse.dtype != torch.float32:
        raise ValueError("lse must be float32 [B, Hq, Nq]")
    if k.dtype != q.dtype or v.dtype != q.dtype or o.dtype != q.dtype:
        raise TypeError("q, k, v and o must share one dtype")
    code = _dtype_code(q)
    _check_cuda(q.device, q=q, k=k, v=v, o=o, lse=lse)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    with torch.cuda.device(q.device):
        if Nk == Nq and Hkv == Hq:
            st = fwd_ptr(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Nq, Hq, D,
                         float(scale), causal, code, stream, **debug)
        else:
            if debug:
                raise ValueError("debug hooks exist only for Nq == Nk and Hq == Hkv")
            st = load_library().fa_fwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                           B, Nq, Nk, Hq, Hkv, D, ctypes.c_float(float(scale)), int(bool(causal)),
                                           code, stream)
    if st != FA_OK:
        raise FaError(st, "fa_fwd")


def fwd(q, k, v, scale: float | None = None, causal: bool = False):
    """Exact attention forward. Returns (o [B,Nq,Hq,D] like q, lse float32 [B,Hq,Nq])."""
    import torch

    B, Nq, Hq, D = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    fwd_into(q, k, v, o, lse, scale=scale, causal=causal)
    return o, lse


def fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, scale: float | None = None,
               causal: bool = False, o=None, lse=None):
    """Forward over packed sequences: q [total_q, Hq, D], k/v [total_k, Hkv, D],
    cu_seqlens_* int32 CUDA tensors of B+1 offsets. Returns (o like q, lse fp32 [Hq, total_q]).
    Inconsistent offsets are reported by status_sync() as FA_ERR_INVALID_ARG."""
    import torch

    if q.dim() != 3 or k.dim() != 3 or v.shape != k.shape or q.shape[2] != k.shape[2]:
        raise ValueError("q must be [total_q, Hq, D] and k, v [total_k, Hkv, D]")
    total_q, Hq, D = q.shape
    total_k, Hkv, _ = k.shape
    if cu_seqlens_q.dtype != torch.int32 or cu_seqlens_k.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    if cu_seqlens_q.dim() != 1 or cu_seqlens_k.shape != cu_seqlens_q.shape:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must be 1-D with B+1 entries")
    B = cu_seqlens_q.numel() - 1
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k and v must share one dtype")
    _dtype_code(q)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device)
    _check_like("o", o, q.shape, q.dtype)
    _check_like("lse", lse, (Hq, total_q), torch.float32)
    _check_cuda(q.device, q=q, k=k, v=v, o=o, lse=lse, cu_seqlens_q=cu_seqlens_q, cu_seqlens_k=cu_seqlens_k)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    with torch.cuda.device(q.device):
        st = load_library().fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                          cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), B, int(max_seqlen_q),
                                          total_q, total_k, Hq, Hkv, D, ctypes.c_float(float(scale)),
                                          int(bool(causal)), _dtype_code(q), stream)
    if st != FA_OK:
        raise FaError(st, "fa_fwd_varlen")
    return o, lse


def splitkv_plan(B: int, Nq: int, Nk: int, Hq: int, D: int, num_splits: int = 0, Hkv: int | None = None) -> tuple[int, int]:
    """(number of key ranges, workspace bytes) fa_fwd_splitkv uses for these sizes on the current device.
    ``Hkv`` (default Hq) selects the packed-heads grid when Nq * Hq / Hkv <= 128."""
    n = ctypes.c_int(0)
    size = ctypes.c_size_t(0)
    hkv = Hq if Hkv is None else Hkv
    st = load_library().fa_fwd_splitkv_plan(B, Nq, Nk, Hq, hkv, D, int(num_splits), ctypes.byref(n),
                                            ctypes.byref(size))
    if st != FA_OK:
        raise FaError(st, "fa_fwd_splitkv_plan")
    return n.value, size.value


def fwd_splitkv(q, k, v, scale: float | None = None, causal: bool = False, num_splits: int = 0, workspace=None,
                o=None, lse=None):
    """Split-KV forward (decode shapes): q [B,Nq,Hq,D], k/v [B,Nk,Hkv,D].

    ``workspace`` is a CUDA uint8 tensor of at least splitkv_plan(...)[1] bytes
    (allocated here with torch if omitted). Returns (o, lse) as fwd does.
    """
    import torch

    _check_qkv4(q, k, v)
    B, Nq, Hq, D = q.shape
    _, Nk, Hkv, _ = k.shape
    if o is not None:
        _check_like("o", o, q.shape, q.dtype)
    if lse is not None:
        _check_like("lse", lse, (B, Hq, Nq), torch.float32)
    if workspace is not None and workspace.dtype != torch.uint8:
        raise TypeError("workspace must be a uint8 tensor")
    _check_cuda(q.device, q=q, k=k, v=v)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    with torch.cuda.device(q.device):
        _, need = splitkv_plan(B, Nq, Nk, Hq, D, num_splits, Hkv=Hkv)
        if workspace is None:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
        if o is None:
            o = torch.empty_like(q)
        if lse is None:
            lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
        _check_cuda(q.device, o=o, lse=lse, workspace=workspace)
        stream = torch.cuda.current_stream(q.device).cuda_stream
        st = load_library().fa_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                           B, Nq, Nk, Hq, Hkv, D, ctypes.c_float(float(scale)), int(bool(causal)),
                                           _dtype_code(q), int(num_splits), workspace.data_ptr(),
                                           workspace.numel() * workspace.element_size(), stream)
    if st != FA_OK:
        raise FaError(st, "fa_fwd_splitkv")
    return o, lse


NOALLOC_SCRATCH_BYTES = 16 << 20  # FA_NOALLOC_SCRATCH_BYTES in include/fa.h


def fwd_splitkv_noalloc(q, k, v, o, lse, scale: float | None = None, causal: bool = False, num_splits: int = 0):
    """Split-KV forward whose partial results use the library's built-in scratch
    buffer instead of a caller workspace, so the call allocates no device memory
    (for callers that cannot allocate on the call path). ``o`` and ``lse`` are
    caller-provided as in fwd_into. Calls overlapping on the GPU share the
    scratch and race; sizes needing more than NOALLOC_SCRATCH_BYTES of partial
    results raise FaError(FA_ERR_UNSUPPORTED)."""
    import torch

    _check_qkv4(q, k, v)
    B, Nq, Hq, D = q.shape
    _, Nk, Hkv, _ = k.shape
    _check_like("o", o, q.shape, q.dtype)
    _check_like("lse", lse, (B, Hq, Nq), torch.float32)
    _check_cuda(q.device, q=q, k=k, v=v, o=o, lse=lse)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    with torch.cuda.device(q.device):
        st = load_library().fa_fwd_splitkv_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                                   lse.data_ptr(), B, Nq, Nk, Hq, Hkv, D, ctypes.c_float(float(scale)),
                                                   int(bool(causal)), _dtype_code(q), int(num_splits), stream)
    if st != FA_OK:
        raise FaError(st, "fa_fwd_splitkv_noalloc")


def bwd_workspace_size(B: int, N: int, H: int) -> int:
    """Device workspace bytes fa_bwd needs for these sizes."""
    size = ctypes.c_size_t(0)
    st = load_library().fa_bwd_workspace_size(int(B), int(N), int(H), ctypes.byref(size))
    if st != FA_OK:
        raise FaError(st, "fa_bwd_workspace_size")
    return size.value


def bwd(q, k, v, o, lse, dout, scale: float | None = None, causal: bool = False, dq=None, dk=None, dv=None,
        workspace=None):
    """Gradients (dq, dk, dv) of sum(O * dout) for the forward's q [B,Nq,Hq,D], k, v [B,Nk,Hkv,D], o and lse.

    ``o`` and ``lse`` are what fwd returned for the same q, k, v, scale and
    causal (with Nk != Nq the causal mask is aligned at the bottom-right
    corner; with Hkv < Hq a K/V head's gradient sums over the query heads that
    read it). dq (like q), dk, dv (like k) and ``workspace`` (CUDA uint8, at
    least bwd_workspace_size(B, Nq, Hq) bytes) are allocated here if omitted.
    """
    import torch

    if q.dim() != 4 or k.dim() != 4 or v.shape != k.shape or o.shape != q.shape or dout.shape != q.shape:
        raise ValueError("q, o, dout must be [B, Nq, Hq, D] and k, v [B, Nk, Hkv, D]")
    B, Nq, Hq, D = q.shape
    Bk, Nk, Hkv, Dk = k.shape
    if Bk != B or Dk != D:
        raise ValueError("q and k/v disagree on batch or head dimension")
    if tuple(lse.shape) != (B, Hq, Nq) or lse.dtype != torch.float32:
        raise ValueError("lse must be float32 [B, Hq, Nq]")
    for t in (k, v, o, dout):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v, o and dout must share one dtype")
    code = _dtype_code(q)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(k) if dv is None else dv
    if dq.shape != q.shape or dq.dtype != q.dtype or dk.shape != k.shape or dv.shape != k.shape or \
            dk.dtype != q.dtype or dv.dtype != q.dtype:
        raise ValueError("dq must be like q, dk and dv like k")
    with torch.cuda.device(q.device):
        need = bwd_workspace_size(B, Nq, Hq)
        if workspace is None:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
        _check_cuda(q.device, q=q, k=k, v=v, o=o, lse=lse, dout=dout, dq=dq, dk=dk, dv=dv, workspace=workspace)
        stream = torch.cuda.current_stream(q.device).cuda_stream
        args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), dout.data_ptr(),
                dq.data_ptr(), dk.data_ptr(), dv.data_ptr())
        tail = (ctypes.c_float(float(scale)), int(bool(causal)), code, workspace.data_ptr(),
                workspace.numel() * workspace.element_size(), stream)
        if Nq == Nk and Hq == Hkv:
            st = load_library().fa_bwd(*args, B, Nq, Hq, D, *tail)
        else:
            st = load_library().fa_bwd_gqa(*args, B, Nq, Nk, Hq, Hkv, D, *tail)
    if st != FA_OK:
        raise FaError(st, "fa_bwd")
    return dq, dk, dv


def bwd_varlen(q, k, v, o, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
               scale: float | None = None, causal: bool = False, dq=None, dk=None, dv=None, workspace=None):
    """Backward of fwd_varlen: q, o, dout [total_q, Hq, D]; k, v [total_k, Hkv, D];
    lse fp32 [Hq, total_q] as fwd_varlen returned it; cu_seqlens_* int32 CUDA
    tensors of B+1 offsets. Returns (dq like q, dk and dv like k). Inconsistent
    offsets are reported by status_sync() as FA_ERR_INVALID_ARG."""
    import torch

    if q.dim() != 3 or k.dim() != 3 or v.shape != k.shape or o.shape != q.shape or dout.shape != q.shape or \
            q.shape[2] != k.shape[2]:
        raise ValueError("q, o, dout must be [total_q, Hq, D] and k, v [total_k, Hkv, D]")
    total_q, Hq, D = q.shape
    total_k, Hkv, _ = k.shape
    if tuple(lse.shape) != (Hq, total_q) or lse.dtype != torch.float32:
        raise ValueError("lse must be float32 [Hq, total_q]")
    if cu_seqlens_q.dtype != torch.int32 or cu_seqlens_k.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    if cu_seqlens_q.dim() != 1 or cu_seqlens_k.shape != cu_seqlens_q.shape:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must be 1-D with B+1 entries")
    for t in (k, v, o, dout):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v, o and dout must share one dtype")
    B = cu_seqlens_q.numel() - 1
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    _dtype_code(q)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(k) if dv is None else dv
    _check_like("dq", dq, q.shape, q.dtype)
    _check_like("dk", dk, k.shape, q.dtype)
    _check_like("dv", dv, k.shape, q.dtype)
    if workspace is not None and workspace.dtype != torch.uint8:
        raise TypeError("workspace must be a uint8 tensor")
    with torch.cuda.device(q.device):
        need = bwd_workspace_size(B, max_seqlen_q, Hq)
        if workspace is None:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
        _check_cuda(q.device, q=q, k=k, v=v, o=o, lse=lse, dout=dout, dq=dq, dk=dk, dv=dv, workspace=workspace,
                    cu_seqlens_q=cu_seqlens_q, cu_seqlens_k=cu_seqlens_k)
        stream = torch.cuda.current_stream(q.device).cuda_stream
        st = load_library().fa_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                          dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                          cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), B, int(max_seqlen_q),
                                          int(max_seqlen_k), total_q, total_k, Hq, Hkv, D,
                                          ctypes.c_float(float(scale)), int(bool(causal)), _dtype_code(q),
                                          workspace.data_ptr(), workspace.numel() * workspace.element_size(), stream)
    if st != FA_OK:
        raise FaError(st, "fa_bwd_varlen")
    return dq, dk, dv
