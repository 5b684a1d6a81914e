"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/fa.h declares, and rejects bad arguments before it
touches a device (no launch, error code returned)."""

import os
import re

import pytest

import exact_attention_151_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "fa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = fa.load_library()
    syms = declared_symbols()
    assert syms == sorted(fa.EXPORTED_SYMBOLS)
    for s in syms:
        assert hasattr(lib, s), s


def test_checking_build_exports_every_declared_symbol():
    lib = fa.load_checking_library()
    for s in declared_symbols():
        assert hasattr(lib, s), s


def test_status_strings():
    for code in range(7):
        assert fa.status_string(code).startswith("FA_")
    assert "UNKNOWN" in fa.status_string(99)


# Argument combinations that must fail validation before any device call.
P = 1 << 20  # a 16-byte aligned, never dereferenced address


@pytest.mark.parametrize("args,expect", [
    ((0, P, P, P, P, 1, 16, 1, 64), fa.FA_ERR_INVALID_ARG),       # null q
    ((P, P, P, P, 0, 1, 16, 1, 64), fa.FA_ERR_INVALID_ARG),       # null lse
    ((P, P, P, P, P, -1, 16, 1, 64), fa.FA_ERR_INVALID_ARG),      # negative B
    ((P, P, P, P, P, 1, -16, 1, 64), fa.FA_ERR_INVALID_ARG),      # negative N
    ((P, P, P, P, P, 1, 16, 1, 96), fa.FA_ERR_UNSUPPORTED),       # D = 96
    ((P, P, P, P, P, 1, 16, 1, 256), fa.FA_ERR_UNSUPPORTED),      # D = 256
    ((P + 8, P, P, P, P, 1, 16, 1, 64), fa.FA_ERR_MISALIGNED),    # q not 16-byte aligned
    ((P, P, P, P, P + 4, 1, 16, 1, 64), fa.FA_ERR_MISALIGNED),    # lse not 16-byte aligned
    ((0, 0, 0, 0, 0, 0, 16, 1, 64), fa.FA_OK),                    # empty batch: no-op
    ((0, 0, 0, 0, 0, 1, 0, 1, 64), fa.FA_OK),                     # empty sequence: no-op
    ((0, 0, 0, 0, 0, 1, 16, 0, 64), fa.FA_OK),                    # no heads: no-op
])
def test_argument_validation(args, expect):
    assert fa.fwd_ptr(*args, 0.125, False, fa.FA_BF16, 0) == expect


def test_bad_dtype_and_scale():
    assert fa.fwd_ptr(P, P, P, P, P, 1, 16, 1, 64, 0.125, False, 7, 0) == fa.FA_ERR_INVALID_ARG
    assert fa.fwd_ptr(P, P, P, P, P, 1, 16, 1, 64, float("inf"), False, fa.FA_BF16, 0) == fa.FA_ERR_INVALID_ARG
    assert fa.fwd_ptr(P, P, P, P, P, 1, 16, 1, 64, float("nan"), True, fa.FA_FP16, 0) == fa.FA_ERR_INVALID_ARG


def test_general_entry_points_validate_before_any_device_call():
    lib = fa.load_library()
    f32 = __import__("ctypes").c_float
    # Hq not a multiple of Hkv
    assert lib.fa_fwd_gqa(P, P, P, P, P, 1, 16, 32, 6, 4, 64, f32(0.1), 0, fa.FA_BF16, 0) == fa.FA_ERR_INVALID_ARG
    # no key/value heads
    assert lib.fa_fwd_gqa(P, P, P, P, P, 1, 16, 32, 6, 0, 64, f32(0.1), 0, fa.FA_BF16, 0) == fa.FA_ERR_INVALID_ARG
    # negative key length
    assert lib.fa_fwd_gqa(P, P, P, P, P, 1, 16, -1, 4, 4, 64, f32(0.1), 0, fa.FA_BF16, 0) == fa.FA_ERR_INVALID_ARG
    # empty query side is a no-op
    assert lib.fa_fwd_gqa(0, 0, 0, 0, 0, 1, 0, 32, 4, 4, 64, f32(0.1), 0, fa.FA_BF16, 0) == fa.FA_OK
    # varlen without offsets
    assert lib.fa_fwd_varlen(P, P, P, P, P, 0, 0, 2, 16, 32, 32, 4, 4, 64, f32(0.1), 0, fa.FA_BF16, 0) == \
        fa.FA_ERR_INVALID_ARG
    # varlen with misaligned output
    assert lib.fa_fwd_varlen(P, P, P, P + 2, P, P, P, 2, 16, 32, 32, 4, 4, 64, f32(0.1), 0, fa.FA_BF16, 0) == \
        fa.FA_ERR_MISALIGNED
    # varlen head dim not supported
    assert lib.fa_fwd_varlen(P, P, P, P, P, P, P, 2, 16, 32, 32, 4, 4, 96, f32(0.1), 0, fa.FA_BF16, 0) == \
        fa.FA_ERR_UNSUPPORTED


def _bwd(lib, q=P, o=P, lse=P, dq=P, ws=P, B=1, N=16, H=1, D=64, scale=0.125, dtype=fa.FA_BF16, ws_bytes=1 << 20):
    f32 = __import__("ctypes").c_float
    return lib.fa_bwd(q, P, P, o, lse, P, dq, P, P, B, N, H, D, f32(scale), 0, dtype, ws, ws_bytes, 0)


def test_backward_validates_before_any_device_call():
    lib = fa.load_library()
    assert _bwd(lib, q=0) == fa.FA_ERR_INVALID_ARG
    assert _bwd(lib, dq=0) == fa.FA_ERR_INVALID_ARG
    assert _bwd(lib, ws=0) == fa.FA_ERR_INVALID_ARG
    assert _bwd(lib, ws_bytes=16) == fa.FA_ERR_INVALID_ARG            # workspace too small
    assert _bwd(lib, B=-1) == fa.FA_ERR_INVALID_ARG
    assert _bwd(lib, dtype=9) == fa.FA_ERR_INVALID_ARG
    assert _bwd(lib, scale=float("nan")) == fa.FA_ERR_INVALID_ARG
    assert _bwd(lib, D=96) == fa.FA_ERR_UNSUPPORTED
    assert _bwd(lib, o=P + 8) == fa.FA_ERR_MISALIGNED
    assert _bwd(lib, ws=P + 16) == fa.FA_ERR_MISALIGNED                # workspace must be 256-byte aligned
    assert _bwd(lib, q=0, o=0, lse=0, dq=0, ws=0, N=0) == fa.FA_OK    # empty: no-op


def test_backward_workspace_size():
    # two fp32 arrays [B*H, N rounded up to 128], each rounded up to 256 bytes,
    # then 256 bytes of work-item counters
    assert fa.bwd_workspace_size(2, 300, 3) == 2 * (2 * 3 * 384 * 4) + 256
    assert fa.bwd_workspace_size(1, 1, 1) == 2 * 512 + 256
    assert fa.bwd_workspace_size(2, 0, 3) == 256  # no queries: the key side still runs (zero dK, dV)
    assert fa.bwd_workspace_size(0, 5, 5) == 0
    lib = fa.load_library()
    import ctypes
    size = ctypes.c_size_t(0)
    assert lib.fa_bwd_workspace_size(-1, 5, 5, ctypes.byref(size)) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_bwd_workspace_size(1, 5, 5, None) == fa.FA_ERR_INVALID_ARG


@pytest.mark.parametrize("B,Nq,Nk,Hq,Hkv,D", [
    (1, 1, 32768, 32, 8, 128), (8, 1, 8192, 32, 8, 128), (1, 1, 4096, 32, 8, 128), (2, 1, 1000, 8, 1, 128),
    (1, 16, 8192, 8, 2, 128), (3, 2, 777, 16, 4, 64), (1, 64, 20000, 4, 4, 128), (1, 300, 2048, 2, 2, 128),
])
def test_splitkv_plan_fits_one_wave(B, Nq, Nk, Hq, Hkv, D):
    """The automatic plan keeps every key range non-empty and the CTAs within one
    wave of 148 SMs; with packed heads (Nq * G <= 128, G > 1) a CTA takes two
    ranges, so the CTA count is half the range count per (batch, K/V head)."""
    splits, ws = fa.splitkv_plan(B, Nq, Nk, Hq, D, 0, Hkv=Hkv)
    n_kt = -(-Nk // 128)
    G = Hq // Hkv
    packed = G > 1 and Nq * G <= 128
    assert 1 <= splits <= min(n_kt, 64)
    tiles = -(-n_kt // splits)
    assert (splits - 1) * tiles < n_kt  # the last range is not empty
    if packed:
        ctas = B * Hkv * (-(-splits // 2) if splits > 1 else 1)
    else:
        ctas = B * Hq * (-(-Nq // 256)) * splits
    assert splits == 1 or ctas <= 148
    assert (ws > 0) == (splits > 1)


def test_noalloc_scratch_has_a_fitting_range_count():
    """Packed heads double the automatic range count, so some plans outgrow the
    no-allocation scratch; fa_fwd_splitkv_noalloc then falls back to the largest
    smaller count that fits, which always exists (one range needs none)."""
    scratch = 16 << 20
    B, Nq, Nk, Hq, Hkv, D = 1, 16, 65536, 32, 4, 128
    splits, need = fa.splitkv_plan(B, Nq, Nk, Hq, D, 0, Hkv=Hkv)
    assert need > scratch
    fits = [r for r in range(splits - 1, 0, -1) if fa.splitkv_plan(B, Nq, Nk, Hq, D, r, Hkv=Hkv)[1] <= scratch]
    assert fits and fa.splitkv_plan(B, Nq, Nk, Hq, D, fits[0], Hkv=Hkv)[0] > 1
