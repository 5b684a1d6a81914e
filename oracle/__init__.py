"""Test infrastructure, not product code: the fp64 CPU oracle.

A thin ctypes wrapper over ``attention_oracle.cpp`` (plain C++17, fp64,
std::thread over rows). Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package; the CUDA
library and its Python binding never do.

What the oracle computes is written out at the top of the C++ file: the
plain definition softmax(scale * Q K^T [+ causal]) V with per-row natural
log-sum-exp (llmtrend.com page, self-attention formula section; tuning
handbook chapter 3, "where the MHA memory bottleneck is"), plus the
handbook's tiled online-softmax routine ("engineering implementation"
section) as an independent second statement.

Inputs are numpy ``uint16`` arrays holding the raw bf16 / fp16 bit patterns
in [B, N, H, D] order, so the oracle sees exactly the bytes the GPU sees.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attention_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

DTYPE_CODES = {"bf16": 0, "fp16": 1}

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (-O2, strict IEEE fp64; no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["g++", "-std=c++17", "-O2", "-fno-fast-math", "-ffp-contract=off", "-shared", "-fPIC",
               "-pthread", _SRC, "-o", _LIB_PATH]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        f64p = ctypes.POINTER(ctypes.c_double)
        i64 = ctypes.c_int64
        i64p = ctypes.POINTER(ctypes.c_int64)
        lib.oracle_decode16.argtypes = [u16p, i64, ctypes.c_int, f64p]
        lib.oracle_decode16.restype = ctypes.c_int
        common = [u16p, u16p, u16p, i64, i64, i64, i64, ctypes.c_double, ctypes.c_int, ctypes.c_int]
        lib.oracle_attention_full.argtypes = common + [f64p, f64p, ctypes.c_int]
        lib.oracle_attention_full.restype = ctypes.c_int
        lib.oracle_attention_rows.argtypes = common + [i64p, i64, f64p, f64p, ctypes.c_int]
        lib.oracle_attention_rows.restype = ctypes.c_int
        lib.oracle_tiled_reference.argtypes = common + [i64, f64p, f64p]
        lib.oracle_tiled_reference.restype = ctypes.c_int
        lib.oracle_attention_varlen.argtypes = [u16p, u16p, u16p, i64p, i64p, i64, i64, i64, i64, ctypes.c_double,
                                                ctypes.c_int, ctypes.c_int, f64p, f64p, ctypes.c_int]
        lib.oracle_attention_varlen.restype = ctypes.c_int
        lib.oracle_attention_backward.argtypes = [u16p, u16p, u16p, u16p, i64, i64, i64, i64, ctypes.c_double,
                                                  ctypes.c_int, ctypes.c_int, f64p, f64p, f64p, ctypes.c_int]
        lib.oracle_attention_backward.restype = ctypes.c_int
        lib.oracle_attention_backward_varlen.argtypes = [u16p, u16p, u16p, u16p, i64p, i64p, i64, i64, i64, i64,
                                                         ctypes.c_double, ctypes.c_int, ctypes.c_int, f64p, f64p,
                                                         f64p, ctypes.c_int]
        lib.oracle_attention_backward_varlen.restype = ctypes.c_int
        _lib = lib
    return _lib


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are raw 16-bit patterns (numpy uint16)")
    return a


def _ptr(a: np.ndarray, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def default_threads() -> int:
    return os.cpu_count() or 1


def decode16(bits, dtype: str) -> np.ndarray:
    """Exact widening of bf16 / fp16 bit patterns to float64."""
    bits = _u16(bits)
    out = np.empty(bits.shape, dtype=np.float64)
    rc = _load().oracle_decode16(_ptr(bits, ctypes.c_uint16), bits.size, DTYPE_CODES[dtype],
                                 _ptr(out, ctypes.c_double))
    if rc:
        raise ValueError(f"oracle_decode16 failed ({rc})")
    return out


def _shape(q, k, v):
    if q.ndim != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share one [B, N, H, D] shape")
    return q.shape


def attention(q, k, v, scale: float, causal: bool, dtype: str, nthreads: int | None = None):
    """The definition with whole score matrices materialised.

    Returns (O [B,N,H,D] float64, LSE [B,H,N] float64).
    """
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, N, H, D = _shape(q, k, v)
    o = np.empty((B, N, H, D), dtype=np.float64)
    lse = np.empty((B, H, N), dtype=np.float64)
    rc = _load().oracle_attention_full(
        _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16), _ptr(v, ctypes.c_uint16), B, N, H, D,
        float(scale), int(bool(causal)), DTYPE_CODES[dtype], _ptr(o, ctypes.c_double),
        _ptr(lse, ctypes.c_double), int(nthreads or default_threads()))
    if rc:
        raise ValueError(f"oracle_attention_full failed ({rc})")
    return o, lse


def attention_rows(q, k, v, scale: float, causal: bool, dtype: str, rows, nthreads: int | None = None):
    """The definition for selected rows; ``rows`` is an int64 array [n, 3] of (b, h, i).

    Returns (O rows [n, D] float64, LSE rows [n] float64).
    """
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, N, H, D = _shape(q, k, v)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    o = np.empty((n, D), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    rc = _load().oracle_attention_rows(
        _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16), _ptr(v, ctypes.c_uint16), B, N, H, D,
        float(scale), int(bool(causal)), DTYPE_CODES[dtype], _ptr(rows, ctypes.c_int64), n,
        _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double), int(nthreads or default_threads()))
    if rc:
        raise ValueError(f"oracle_attention_rows failed ({rc})")
    return o, lse


def attention_varlen(q, k, v, cu_q, cu_k, scale: float, causal: bool, dtype: str, nthreads: int | None = None):
    """Packed sequences with grouped-query heads and bottom-right causal alignment.

    q: [total_q, Hq, D], k and v: [total_k, Hkv, D] (uint16 patterns); cu_q, cu_k: B+1
    prefix offsets. Returns (O [total_q, Hq, D] float64, LSE [Hq, total_q] float64);
    a query with no visible key has O = 0 and LSE = -inf.
    """
    q, k, v = _u16(q), _u16(k), _u16(v)
    if q.ndim != 3 or k.ndim != 3 or k.shape != v.shape or q.shape[2] != k.shape[2]:
        raise ValueError("q must be [total_q, Hq, D], k and v [total_k, Hkv, D]")
    cu_q = np.ascontiguousarray(np.asarray(cu_q, dtype=np.int64))
    cu_k = np.ascontiguousarray(np.asarray(cu_k, dtype=np.int64))
    B = len(cu_q) - 1
    if len(cu_k) != B + 1 or cu_q[-1] != q.shape[0] or cu_k[-1] != k.shape[0]:
        raise ValueError("cu_seqlens do not match the tensors")
    total_q, Hq, D = q.shape
    Hkv = k.shape[1]
    o = np.empty((total_q, Hq, D), dtype=np.float64)
    lse = np.empty((Hq, total_q), dtype=np.float64)
    rc = _load().oracle_attention_varlen(
        _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16), _ptr(v, ctypes.c_uint16), _ptr(cu_q, ctypes.c_int64),
        _ptr(cu_k, ctypes.c_int64), B, Hq, Hkv, D, float(scale), int(bool(causal)), DTYPE_CODES[dtype],
        _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double), int(nthreads or default_threads()))
    if rc:
        raise ValueError(f"oracle_attention_varlen failed ({rc})")
    return o, lse


def attention_backward(q, k, v, dout, scale: float, causal: bool, dtype: str, nthreads: int | None = None):
    """Gradients (dQ, dK, dV), float64 [B, N, H, D], of sum(O * dO) through the
    definition; all inputs are 16-bit patterns in [B, N, H, D]."""
    q, k, v, dout = _u16(q), _u16(k), _u16(v), _u16(dout)
    B, N, H, D = _shape(q, k, v)
    if dout.shape != q.shape:
        raise ValueError("dO must match q")
    dq = np.empty((B, N, H, D), dtype=np.float64)
    dk = np.empty_like(dq)
    dv = np.empty_like(dq)
    rc = _load().oracle_attention_backward(
        _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16), _ptr(v, ctypes.c_uint16), _ptr(dout, ctypes.c_uint16),
        B, N, H, D, float(scale), int(bool(causal)), DTYPE_CODES[dtype], _ptr(dq, ctypes.c_double),
        _ptr(dk, ctypes.c_double), _ptr(dv, ctypes.c_double), int(nthreads or default_threads()))
    if rc:
        raise ValueError(f"oracle_attention_backward failed ({rc})")
    return dq, dk, dv


def attention_backward_varlen(q, k, v, dout, cu_q, cu_k, scale: float, causal: bool, dtype: str,
                              nthreads: int | None = None):
    """Gradients (dQ [total_q, Hq, D], dK and dV [total_k, Hkv, D], float64) of
    sum(O * dO) through attention_varlen's definition: packed sequences,
    grouped-query heads (a K/V head's gradient sums over the query heads that
    read it), causal mask aligned at the bottom-right corner. Inputs are 16-bit
    patterns: q and dout [total_q, Hq, D], k and v [total_k, Hkv, D]."""
    q, k, v, dout = _u16(q), _u16(k), _u16(v), _u16(dout)
    if q.ndim != 3 or k.ndim != 3 or k.shape != v.shape or q.shape[2] != k.shape[2] or dout.shape != q.shape:
        raise ValueError("q and dout must be [total_q, Hq, D], k and v [total_k, Hkv, D]")
    cu_q = np.ascontiguousarray(np.asarray(cu_q, dtype=np.int64))
    cu_k = np.ascontiguousarray(np.asarray(cu_k, dtype=np.int64))
    B = len(cu_q) - 1
    if len(cu_k) != B + 1 or cu_q[-1] != q.shape[0] or cu_k[-1] != k.shape[0]:
        raise ValueError("cu_seqlens do not match the tensors")
    total_q, Hq, D = q.shape
    Hkv = k.shape[1]
    dq = np.empty((total_q, Hq, D), dtype=np.float64)
    dk = np.empty(k.shape, dtype=np.float64)
    dv = np.empty(k.shape, dtype=np.float64)
    rc = _load().oracle_attention_backward_varlen(
        _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16), _ptr(v, ctypes.c_uint16), _ptr(dout, ctypes.c_uint16),
        _ptr(cu_q, ctypes.c_int64), _ptr(cu_k, ctypes.c_int64), B, Hq, Hkv, D, float(scale), int(bool(causal)),
        DTYPE_CODES[dtype], _ptr(dq, ctypes.c_double), _ptr(dk, ctypes.c_double), _ptr(dv, ctypes.c_double),
        int(nthreads or default_threads()))
    if rc:
        raise ValueError(f"oracle_attention_backward_varlen failed ({rc})")
    return dq, dk, dv


def tiled_reference(q, k, v, scale: float, causal: bool, dtype: str, block_size: int = 128):
    """The handbook's tiled online-softmax routine in fp64 (single thread)."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, N, H, D = _shape(q, k, v)
    o = np.empty((B, N, H, D), dtype=np.float64)
    lse = np.empty((B, H, N), dtype=np.float64)
    rc = _load().oracle_tiled_reference(
        _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16), _ptr(v, ctypes.c_uint16), B, N, H, D,
        float(scale), int(bool(causal)), DTYPE_CODES[dtype], int(block_size), _ptr(o, ctypes.c_double),
        _ptr(lse, ctypes.c_double))
    if rc:
        raise ValueError(f"oracle_tiled_reference failed ({rc})")
    return o, lse
