"""Parity metrics between the CUDA path and the fp64 oracle (test infrastructure).

Tolerances (16-bit inputs, fp32 accumulation on the GPU):
  max |O_gpu - O_ref|              <= 1e-2
  ||O_gpu - O_ref||_2 / ||O_ref||_2 <= 5e-3
  max |LSE_gpu - LSE_ref|          <= 1e-3
"""

from __future__ import annotations

import numpy as np

TOL_MAX_ABS_O = 1e-2
TOL_REL_L2_O = 5e-3
TOL_MAX_ABS_LSE = 1e-3


def metrics(o_gpu, lse_gpu, o_ref, lse_ref) -> dict:
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
    lse_ref = np.asarray(lse_ref, dtype=np.float64)
    diff = o_gpu - o_ref
    ref_norm = float(np.linalg.norm(o_ref))
    return {
        "max_abs_o": float(np.abs(diff).max()) if diff.size else 0.0,
        "rel_l2_o": float(np.linalg.norm(diff) / ref_norm) if ref_norm > 0 else float(np.linalg.norm(diff)),
        "max_abs_lse": float(np.abs(lse_gpu - lse_ref).max()) if lse_ref.size else 0.0,
        "finite": bool(np.isfinite(o_gpu).all() and np.isfinite(lse_gpu).all()),
    }


def passes(m: dict) -> bool:
    return (m["finite"] and m["max_abs_o"] <= TOL_MAX_ABS_O and m["rel_l2_o"] <= TOL_REL_L2_O
            and m["max_abs_lse"] <= TOL_MAX_ABS_LSE)


def sample_rows(B: int, H: int, N: int, per_head_random: int, seed: int = 0, heads: list | None = None,
                block: int = 128, ends: int = 2) -> np.ndarray:
    """(b, h, i) triples covering, for each chosen head (default: every head),
    the first and last `ends` rows, the rows on both sides of every `block`
    boundary, and `per_head_random` random rows."""
    rng = np.random.default_rng(seed)
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(H)]
    edge = set(range(min(ends, N))) | set(range(max(0, N - ends), N))
    for t in range(block, N, block):
        edge.update((t - 1, t))
    edge = sorted(i for i in edge if 0 <= i < N)
    out = []
    for b, h in heads:
        rows = set(edge)
        rows.update(rng.integers(0, N, size=per_head_random).tolist())
        out.extend((b, h, i) for i in sorted(rows))
    return np.array(out, dtype=np.int64)


# Backward (dQ, dK, dV). Each gradient element is a sum of products whose
# 16-bit factor (P or dS, rounded once before the tensor cores) carries a
# relative error up to u (bf16 2^-8, fp16 2^-11), and the result is rounded to
# the same dtype once more: with independent roundings the expected relative
# L2 error is about 0.8 u (3.2e-3 bf16, 4e-4 fp16); the bound allows about 3x
# (bf16) and 4x (fp16) that. The error of one element is about 0.8 u times its
# own scale (the root of the sum of its squared terms), so the largest error
# is compared with the largest reference magnitude: a 5-sigma error on the
# largest-scale elements is about 4 u of that scale, and the bound is 5 u.
# (Relative to the RMS instead, causal gradients would be penalised for the
# spread of their magnitudes: early keys collect terms from many queries.)
TOL_GRAD_REL_L2 = {"bf16": 1e-2, "fp16": 2e-3}
TOL_GRAD_MAX_REL = {"bf16": 5 * 2.0**-8, "fp16": 5 * 2.0**-11}


def grad_metrics(got, ref) -> dict:
    out = {}
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        g = np.asarray(g, dtype=np.float64)
        r = np.asarray(r, dtype=np.float64)
        diff = g - r
        rn = float(np.linalg.norm(r))
        rmax = float(np.abs(r).max(initial=0.0))
        dmax = float(np.abs(diff).max(initial=0.0))
        out[name] = {
            "rel_l2": float(np.linalg.norm(diff) / rn) if rn > 0 else float(np.linalg.norm(diff)),
            "max_rel": dmax / rmax if rmax > 0 else dmax,
            "finite": bool(np.isfinite(g).all()),
        }
    return out


def grad_passes(m: dict, dtype: str) -> bool:
    return all(x["finite"] and x["rel_l2"] <= TOL_GRAD_REL_L2[dtype] and x["max_rel"] <= TOL_GRAD_MAX_REL[dtype]
               for x in m.values())
