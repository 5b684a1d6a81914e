#!/usr/bin/env python
"""Benchmark of the fused exact-attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--pass fwd|bwd] [--shard]

One step = one fa_fwd call over the whole workload (default: the sequence-sweep
point N=32768, B=1 H=16 D=128 bf16 non-causal, the largest single-GPU
configuration and inside the "non-causal, N >= 4k" range the forward's target
is stated on). Prints ONE JSON line on rank 0.

  value      forward TFLOP/s of the whole job (4*B*H*N^2*D per step, halved for
             causal) with inputs resident in HBM; device time from CUDA events
             around exactly K steps (barrier + synchronize on both sides), max
             over ranks. Q+K+V+O (512 MiB at the default) exceed the 126 MB L2,
             so no flush is done between steps.
  e2e        the same metric through the public API with pinned host buffers:
             each step copies Q, K, V host->device, runs fa_fwd and copies O and
             LSE back, all inside the timed region; two buffer sets and three
             streams let the copies of neighbouring steps overlap the kernels.
  roofline   tensor-core bound: achieved TFLOP/s of the kernel against the
             measured cuBLAS bf16 peak; dram traffic per launch from the
             committed ncu summary when it matches the current kernel source.
  cpu_baseline  the fp64 oracle on a bounded row sample, on the host cores
             (rank 0 at N=1 only); the same rows double as a parity check.

--pass bwd times the backward instead (one step = one fa_bwd call: the D/LSE
preprocess, the dQ kernel and the dK/dV kernel), counted as 2.5x the forward's
flops (five N x N x D products against the forward's two); its e2e copies q,
k, v, o, lse and dO in and dQ, dK, dV out, and its cpu_baseline is the oracle's
backward on one (batch, head) slice.

With torchrun (N>1) every rank runs the full workload on its own GPU by
default (weak scaling: the job is N independent copies of the workload, no
collective on the data path); the timing is reduced with MAX. --shard splits
ONE workload over the ranks instead (contiguous batch slices, or head slices
when B < N) and ends every step with an NCCL all-gather of O and LSE, so each
rank holds the whole result (strong scaling).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd TFLOPS (bf16, d=128) and % of B200 dense tensor peak"
METRIC_BWD = "attention bwd TFLOPS (bf16, d=128) and % of B200 dense tensor peak"
BWD_FLOP_FACTOR = 2.5  # backward flops per forward flop (5 vs 2 matrix products)
DEFAULT_WORKLOAD = "sweep_n32768_noncausal"
KERNEL_SOURCES = [os.path.join(ROOT, "exact_attention_151_b200", "csrc", f) for f in ("fa_fwd.cu", "fa_fwd_kernel.cuh", "sm100.cuh")]
BWD_KERNEL_SOURCES = KERNEL_SOURCES + [os.path.join(ROOT, "exact_attention_151_b200", "csrc", "fa_bwd_kernel.cuh")]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK_PEAK_TFLOPS = 1590.0


def kernel_source_hash(sources=None) -> str:
    h = hashlib.sha256()
    for p in sources or KERNEL_SOURCES:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_PEAK_TFLOPS, 1400.0, "fallback"


def measured_hbm() -> float:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"])
    except Exception:
        return 6650.0


def recorded_traffic(workload: str, sources=None):
    """DRAM bytes per launch from the committed ncu summary, if taken on this kernel source."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
        e = d.get(workload)
        if e and e.get("kernel_source_hash") == kernel_source_hash(sources):
            return float(e["dram_bytes_per_launch"]), e.get("how", "")
    except Exception:
        pass
    return None, None


class ClockSampler:
    """Polls NVML (SM clock, throttle reasons) in a thread during the timed region."""

    REASONS = {
        0x0000000000000004: "sw_power_cap",
        0x0000000000000008: "hw_slowdown",
        0x0000000000000020: "sw_thermal_slowdown",
        0x0000000000000040: "hw_thermal_slowdown",
        0x0000000000000080: "hw_power_brake_slowdown",
        0x0000000000000002: "applications_clocks_setting",
    }

    def __init__(self, uuid: str, period_s: float = 0.002):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self.error = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nvml = pynvml
            u = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self._h = pynvml.nvmlDeviceGetHandleByUUID(u.encode() if isinstance(u, str) else u)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report that instead of clocks
            self._nvml = None
            self.error = f"nvml unavailable: {e}"

    def _run(self):
        n = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM))
                r = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception as e:
                self.error = str(e)
                return
            time.sleep(self.period)

    def __enter__(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        d = {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
             "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}
        if self.error:
            d["error"] = self.error
        return d


def row_flops(w, rows) -> float:
    """Algorithmic flops of the sampled rows: 4*D per visible key (QK^T and PV)."""
    import numpy as np

    rows = np.asarray(rows)
    nk, nq = w.n_keys, w.N
    if w.causal:
        nvis = np.clip(rows[:, 2] + nk - nq + 1, 0, nk)
    else:
        nvis = np.full(len(rows), nk)
    return float(4.0 * w.D * nvis.sum())


def is_square(w) -> bool:
    return w.n_keys == w.N and w.kv_heads == w.H


def oracle_row_sample(w, q, k, v, target_s: float, seed: int = 0):
    """Time the oracle on a row sample sized to roughly target_s seconds of host work."""
    import numpy as np

    import oracle
    from exact_attention_151_b200.inputs import bits

    Q, K, V = bits(q), bits(k), bits(v)
    rng = np.random.default_rng(seed)
    threads = oracle.default_threads()
    if not is_square(w):
        # decode-like shapes: the whole (small) query side through the packed form
        B, Nq, Hq, D = q.shape
        Nk, Hkv = k.shape[1], k.shape[2]
        t0 = time.perf_counter()
        o, lse = oracle.attention_varlen(Q.reshape(B * Nq, Hq, D), K.reshape(B * Nk, Hkv, D), V.reshape(B * Nk, Hkv, D),
                                         np.arange(B + 1) * Nq, np.arange(B + 1) * Nk, w.softmax_scale, w.causal,
                                         w.dtype, nthreads=threads)
        dt = time.perf_counter() - t0
        rows = np.array([(b, h, i) for b in range(B) for h in range(Hq) for i in range(Nq)], dtype=np.int64)
        o_rows = o.reshape(B, Nq, Hq, D)[rows[:, 0], rows[:, 2], rows[:, 1]]
        lse_rows = lse.reshape(Hq, B, Nq)[rows[:, 1], rows[:, 0], rows[:, 2]]
        return rows, o_rows, lse_rows, dt, threads

    def draw(n):
        return np.stack([rng.integers(0, w.B, n), rng.integers(0, w.H, n), rng.integers(0, w.N, n)], axis=1)

    probe = draw(max(threads, 8))
    t0 = time.perf_counter()
    oracle.attention_rows(Q, K, V, w.softmax_scale, w.causal, w.dtype, probe, nthreads=threads)
    dt = max(time.perf_counter() - t0, 1e-3)
    n = int(max(threads, min(200000, len(probe) * target_s / dt)))
    rows = draw(n)
    t0 = time.perf_counter()
    o_ref, lse_ref = oracle.attention_rows(Q, K, V, w.softmax_scale, w.causal, w.dtype, rows, nthreads=threads)
    dt = time.perf_counter() - t0
    return rows, o_ref, lse_ref, dt, threads


def run_reference(args, w):
    """The oracle on the host cores, each step a bounded row sample (rank 0 only)."""
    import numpy as np

    from exact_attention_151_b200.inputs import make_qkv

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    q, k, v = make_qkv(w)
    per_step_target = max(1.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    times, flops = [], []
    for i in range(args.warmup + args.steps):
        rows, _, _, dt, threads = oracle_row_sample(w, q, k, v, per_step_target, seed=100 + i)
        if i >= args.warmup:
            times.append(dt)
            flops.append(row_flops(w, rows))
    value = sum(flops) / sum(times) / 1e12
    sample = (f"{len(rows)} random (b,h,i) rows per step of the {w.name} workload "
              f"(~{per_step_target:.0f} s of fp64 work per step)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def bwd_slice_sample(w, q, k, v, dout, target_s: float, seed: int = 0):
    """The oracle's backward on whole (b, h) slices, as many as fit in about target_s seconds (at least one)."""
    import numpy as np

    import oracle
    from exact_attention_151_b200.inputs import bits

    rng = np.random.default_rng(seed)
    threads = oracle.default_threads()
    picks, refs, dt = [], [], 0.0
    while not picks or dt < target_s * 0.5:
        b, h = int(rng.integers(0, w.B)), int(rng.integers(0, w.H))
        sl = (slice(b, b + 1), slice(None), slice(h, h + 1))
        t0 = time.perf_counter()
        refs.append(oracle.attention_backward(bits(q[sl]), bits(k[sl]), bits(v[sl]), bits(dout[sl]), w.softmax_scale,
                                              w.causal, w.dtype, nthreads=threads))
        dt += time.perf_counter() - t0
        picks.append((b, h))
        if len(picks) >= w.B * w.H:
            break
    return picks, refs, dt, threads


def run_reference_bwd(args, w):
    """The oracle's backward on the host cores, each step whole (b, h) slices (rank 0 only)."""
    from exact_attention_151_b200.inputs import make_dout, make_qkv

    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    q, k, v = make_qkv(w)
    dout = make_dout(w)
    per_step_target = max(1.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    slice_flops = BWD_FLOP_FACTOR * w.flops / (w.B * w.H)
    times, flops = [], []
    for i in range(args.warmup + args.steps):
        picks, _, dt, threads = bwd_slice_sample(w, q, k, v, dout, per_step_target, seed=100 + i)
        if i >= args.warmup:
            times.append(dt)
            flops.append(slice_flops * len(picks))
    value = sum(flops) / sum(times) / 1e12
    sample = (f"{len(picks)} whole (b,h) slice(s) of the {w.name} workload's backward per step "
              f"(as many as fit in ~{per_step_target:.0f} s of fp64 work, at most all B*H)")
    line = {
        "impl": "reference", "metric": METRIC_BWD, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": dict(workload_config(w), **{"pass": "backward"}),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_backward(args, w, dev, world, rank):
    """Time fa_bwd (preprocess + dQ kernel + dK/dV kernel) over the whole workload."""
    import torch
    import torch.distributed as dist

    import exact_attention_151_b200 as fa
    from exact_attention_151_b200.inputs import make_dout, make_qkv

    q, k, v = make_qkv(w)
    dout = make_dout(w)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, dout))
    od, lsed = fa.fwd(qd, kd, vd, scale=w.softmax_scale, causal=w.causal)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(qd), torch.empty_like(qd)
    workspace = torch.empty(max(fa.bwd_workspace_size(w.B, w.N, w.H), 1), dtype=torch.uint8, device=dev)
    flops = BWD_FLOP_FACTOR * w.flops
    # bytes a backward must move at least: read q, k, v, o, dO (16-bit) and lse, write dq, dk, dv
    min_bytes = 8 * w.B * w.N * w.H * w.D * 2 + 4 * w.B * w.H * w.N
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev) if min_bytes <= 126e6 else None
    stream = torch.cuda.current_stream(dev)

    def step():
        fa.bwd(qd, kd, vd, od, lsed, dod, scale=w.softmax_scale, causal=w.causal, dq=dq, dk=dk, dv=dv,
               workspace=workspace)

    for _ in range(args.warmup):
        step()
    if fa.status_sync(stream.cuda_stream) != fa.FA_OK:
        raise RuntimeError("device status word reports a timeout during warm-up")
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    with ClockSampler(uuid) as clocks:
        t_start.record(stream)
        for i in range(args.steps):
            if flush is not None:
                flush.zero_()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    if fa.status_sync(stream.cuda_stream) != fa.FA_OK:
        raise RuntimeError("device status word reports a timeout in the timed region")
    launch_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = sum(launch_ms) if flush is not None else t_start.elapsed_time(t_end)
    t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    max_ms = float(t.item())
    value = flops * args.steps * world / (max_ms * 1e-3) / 1e12
    avg_ms = sum(launch_ms) / len(launch_ms)

    # end to end: inputs host->device, backward, gradients device->host (overlapped across steps)
    e2e_steps = args.e2e_steps or max(3, min(args.steps, 20))
    host_in = [t.pin_memory() for t in (q, k, v, od.cpu(), lsed.cpu(), dout)]
    slot0 = {"inputs": [qd, kd, vd, od, lsed, dod], "outputs": [dq, dk, dv]}
    slot1 = {"inputs": [t.clone() for t in slot0["inputs"]], "outputs": [torch.empty_like(t) for t in (dq, dk, dv)]}
    slots = [slot0, slot1]
    for sl in slots:
        sl["host_out"] = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in sl["outputs"]]

    def compute(sl):
        q_, k_, v_, o_, l_, do_ = sl["inputs"]
        dq_, dk_, dv_ = sl["outputs"]
        fa.bwd(q_, k_, v_, o_, l_, do_, scale=w.softmax_scale, causal=w.causal, dq=dq_, dk=dk_, dv=dv_,
               workspace=workspace)

    e2e_ms = pipelined_e2e(dev, e2e_steps, host_in, slots, compute, world)
    h2d = sum(h_.numel() * h_.element_size() for h_ in host_in)
    d2h = sum(h_.numel() * h_.element_size() for h_ in slot0["host_out"])
    e2e_value = flops * e2e_steps * world / (e2e_ms * 1e-3) / 1e12

    if rank == 0:
        peak, peak_sus, peak_src = measured_peak()
        achieved = flops / (avg_ms * 1e-3) / 1e12
        traffic, traffic_how = recorded_traffic(w.name + ":bwd", BWD_KERNEL_SOURCES)
        line = {
            "metric": METRIC_BWD, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": dict(workload_config(w), **{"pass": "backward", "flops_per_step": flops}),
            "pct_of_peak": 100.0 * value / world / peak,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{peak_src} bf16 burst (MEASURED_PEAKS.json bf16_tflops)",
                         "frac_of_sustained_peak": achieved / peak_sus, "algorithmic_bytes": min_bytes,
                         "traffic_source": traffic_how,
                         "note": "achieved and frac: the whole step (preprocess, dQ and dK/dV kernels); traffic: the "
                                 "dominant dK/dV kernel's DRAM bytes per launch"},
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps, "ms_per_step": e2e_ms / e2e_steps,
                    "pcie_gbs": (h2d + d2h) * e2e_steps / (e2e_ms * 1e-3) / 1e9,
                    "overlap": "two buffer sets; host->device copies, kernels and device->host copies on three "
                               "streams"},
            "clocks": clocks.summary(),
            "gpu_launches": args.steps * 3,
            "kernel_source_hash": kernel_source_hash(BWD_KERNEL_SOURCES),
        }
        if world == 1 and not args.no_cpu_baseline:
            from tests.parity import grad_metrics, grad_passes

            picks, refs, dt, threads = bwd_slice_sample(w, q, k, v, dout, args.cpu_seconds)
            grads = [g.cpu().to(torch.float64).numpy() for g in (dq, dk, dv)]
            worst = None
            for (b, h), ref in zip(picks, refs):
                sl = (slice(b, b + 1), slice(None), slice(h, h + 1))
                m = grad_metrics([g[sl] for g in grads], ref)
                if worst is None or max(x["rel_l2"] for x in m.values()) > max(x["rel_l2"] for x in worst.values()):
                    worst = m
            line["cpu_baseline"] = {
                "value": BWD_FLOP_FACTOR * w.flops / (w.B * w.H) * len(picks) / dt / 1e12, "unit": "TFLOP/s",
                "cores": threads, "kind": "oracle",
                "sample": f"{len(picks)} whole (b,h) slices of the same inputs' backward, fp64, {dt:.1f} s"}
            line["parity"] = {"worst_slice": worst, "slices": len(picks),
                              "passes": all(grad_passes(grad_metrics([g[(slice(b, b + 1), slice(None), slice(h, h + 1))]
                                                                      for g in grads], ref), w.dtype)
                                            for (b, h), ref in zip(picks, refs))}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def workload_config(w):
    extra = {} if is_square(w) else {"Nk": w.n_keys, "Hkv": w.kv_heads, "causal_alignment": "bottom-right"}
    if w.splitkv:
        extra["path"] = "split-KV (fa_fwd_splitkv: partial kernel + merge kernel)"
    return {"workload": w.name, "B": w.B, "N": w.N, "H": w.H, "D": w.D, "dtype": w.dtype, "causal": w.causal, **extra,
            "scale": w.softmax_scale, "flops_per_step": w.flops, "seed": w.seed,
            "inputs": f"Q~N(0,{w.q_std}^2) K~N(0,{w.k_std}^2) V~{'U(-1,1)' if w.v_dist == 'uniform' else 'N(0,1)'}",
            "l2": "no flush: Q+K+V+O exceed the 126 MB L2" if w.min_hbm_bytes > 126e6 else
                  "L2 flushed between steps (256 MiB write, outside the per-step kernel events)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--pass", dest="which", default="fwd", choices=["fwd", "bwd"])
    ap.add_argument("--shard", action="store_true",
                    help="split one workload over the ranks (batch or heads) and all-gather O and LSE each step")
    ap.add_argument("--no-graph", action="store_true",
                    help="forward: launch every timed step through the Python API instead of replaying a CUDA graph "
                         "of one step")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    from exact_attention_151_b200.inputs import WORKLOADS

    w = WORKLOADS[args.workload]
    if args.which == "bwd":
        if not is_square(w) or w.splitkv:
            raise SystemExit("--pass bwd needs a square self-attention workload")
        if args.impl == "reference":
            return run_reference_bwd(args, w)
    elif args.impl == "reference":
        return run_reference(args, w)

    import numpy as np
    import torch
    import torch.distributed as dist

    import exact_attention_151_b200 as fa
    from exact_attention_151_b200.inputs import make_qkv

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local_rank))
    dev = torch.device("cuda", local_rank if world > 1 else 0)
    torch.cuda.set_device(dev)
    if args.which == "bwd":
        return run_backward(args, w, dev, world, rank)

    return run_forward(args, w, dev, world, rank)


def pipelined_e2e(dev, n_steps, host_in, slots, compute, world):
    """End-to-end time of n_steps steps through the public API, in ms (max over ranks).

    Every step copies its inputs host->device from pinned buffers (``host_in``),
    runs ``compute(slot)`` and copies the slot's results device->host. Two
    buffer sets (``slots``: dicts with device "inputs", device "outputs" and
    pinned "host_out") alternate, and the copies in, the kernels and the copies
    out run on three streams, so the input copy of step i+1 and the output copy
    of step i-1 overlap the kernels of step i. A slot's inputs are only
    overwritten after the kernels of two steps back have read them, and its
    outputs only after they have been copied out."""
    import torch
    import torch.distributed as dist

    comp, up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    h2d = [torch.cuda.Event() for _ in slots]
    done = [torch.cuda.Event() for _ in slots]
    d2h = [torch.cuda.Event() for _ in slots]

    def one(i):
        s = i % len(slots)
        sl = slots[s]
        up.wait_event(done[s])
        with torch.cuda.stream(up):
            for d_, h_ in zip(sl["inputs"], host_in):
                d_.copy_(h_, non_blocking=True)
        h2d[s].record(up)
        comp.wait_event(h2d[s])
        comp.wait_event(d2h[s])
        with torch.cuda.stream(comp):
            compute(sl)
        done[s].record(comp)
        down.wait_event(done[s])
        with torch.cuda.stream(down):
            for h_, d_ in zip(sl["host_out"], sl["outputs"]):
                h_.copy_(d_, non_blocking=True)
        d2h[s].record(down)

    for i in range(len(slots)):  # warm-up: every event recorded once
        one(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    up.wait_event(e0)
    down.wait_event(e0)
    for i in range(n_steps):
        one(i)
    for ev in d2h:
        comp.wait_event(ev)
    e1.record(comp)
    torch.cuda.synchronize(dev)
    te = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(te, op=dist.ReduceOp.MAX)
        dist.barrier()
    return float(te.item())


def run_forward(args, w, dev, world, rank):
    """Time fa_fwd (or the split-KV pair of kernels) over the workload; with --shard, one workload split
    over the ranks plus the all-gather of O and LSE."""
    import torch
    import torch.distributed as dist

    import exact_attention_151_b200 as fa
    from exact_attention_151_b200.inputs import make_qkv
    from exact_attention_151_b200.sharding import ForwardSharding

    q, k, v = make_qkv(w)
    shard = None
    if args.shard:
        if not is_square(w) or w.splitkv:
            raise SystemExit("--shard needs a square self-attention workload")
        shard = [ForwardSharding(w.B, w.N, w.H, w.D, world, rank, dev, q.dtype) for _ in range(2)]
        q_in, k_in, v_in = (shard[0].local(t) for t in (q, k, v))
    else:
        q_in, k_in, v_in = q, k, v
    lse_shape = shard[0].local_lse_shape() if shard else (w.B, w.H, w.N)

    def make_slot():
        qd_, kd_, vd_ = q_in.to(dev), k_in.to(dev), v_in.to(dev)
        return {"inputs": [qd_, kd_, vd_],
                "o": torch.empty_like(qd_), "lse": torch.empty(lse_shape, dtype=torch.float32, device=dev)}

    slots = [make_slot(), make_slot()]
    flush = None
    if w.min_hbm_bytes <= 126e6:
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    kernels_per_step = 1
    workspace = None
    if w.splitkv:
        n_splits, ws_bytes = fa.splitkv_plan(w.B, w.N, w.n_keys, w.H, w.D, Hkv=w.kv_heads)
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
        kernels_per_step = 2 if n_splits > 1 else 1

    def compute(sl, s_idx=0):
        qd_, kd_, vd_ = sl["inputs"]
        if w.splitkv:
            fa.fwd_splitkv(qd_, kd_, vd_, scale=w.softmax_scale, causal=w.causal, workspace=workspace, o=sl["o"],
                           lse=sl["lse"])
        else:
            fa.fwd_into(qd_, kd_, vd_, sl["o"], sl["lse"], scale=w.softmax_scale, causal=w.causal)
        if shard:
            sl["shard"].exchange(sl["o"], sl["lse"])

    if shard:
        for sl, sh in zip(slots, shard):
            sl["shard"] = sh
            sl["outputs"] = [sh.o_recv, sh.l_recv]
    else:
        for sl in slots:
            sl["outputs"] = [sl["o"], sl["lse"]]
    stream = torch.cuda.current_stream(dev)

    def step():
        compute(slots[0])

    for _ in range(args.warmup):
        step()
    if fa.status_sync(stream.cuda_stream) != fa.FA_OK:
        raise RuntimeError("device status word reports a timeout during warm-up")
    # One step captured as a CUDA graph (the same kernel launches with the same
    # buffers), replayed once per timed step, so that the host's per-call
    # Python and argument marshalling stay off the device timeline; short steps
    # (decode, the small config) are otherwise bound by the host.
    graph = None
    if not args.no_graph and not shard:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        graph.replay()
        torch.cuda.synchronize(dev)
        if fa.status_sync(stream.cuda_stream) != fa.FA_OK:
            raise RuntimeError("device status word reports a timeout in the captured step")

        def step():  # noqa: F811
            graph.replay()

    # ---- timed region: exactly K steps, per-step events on the launching stream
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    with ClockSampler(uuid) as clocks:
        t_start.record(stream)
        for i in range(args.steps):
            if flush is not None:
                flush.zero_()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    if fa.status_sync(stream.cuda_stream) != fa.FA_OK:
        raise RuntimeError("device status word reports a timeout in the timed region")
    total_ms = t_start.elapsed_time(t_end)
    launch_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    if flush is not None:  # the flush writes sit between launches; count only kernel time
        total_ms = sum(launch_ms)
    t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    max_ms = float(t.item())
    ms_per_step = max_ms / args.steps
    # replicas: every rank does the whole workload; --shard: the ranks share one
    job_flops = w.flops * (1 if shard else world)
    value = job_flops * args.steps / (max_ms * 1e-3) / 1e12
    avg_launch_ms = sum(launch_ms) / len(launch_ms)

    # ---- end to end through the public API with pinned host buffers, copies overlapped with the kernels
    e2e_steps = args.e2e_steps or max(3, min(args.steps, 50))
    host_in = [t.pin_memory() for t in (q_in, k_in, v_in)]
    for sl in slots:
        sl["host_out"] = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in sl["outputs"]]
    e2e_ms = pipelined_e2e(dev, e2e_steps, host_in, slots, compute, world)
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in slots[0]["host_out"])
    e2e_value = job_flops * e2e_steps / (e2e_ms * 1e-3) / 1e12

    if rank == 0:
        peak, peak_sus, peak_src = measured_peak()
        kernel_flops = w.flops / world if shard else w.flops
        achieved = kernel_flops / (avg_launch_ms * 1e-3) / 1e12
        traffic, traffic_how = recorded_traffic(w.name)
        intensity = w.flops / w.min_hbm_bytes
        # the kernel's roofline: tensor-bound above the ridge of the measured peaks
        ridge = peak * 1e12 / (measured_hbm() * 1e9)
        cfg = workload_config(w)
        cfg["launch"] = ("a CUDA graph of one step (the same kernel launches), replayed per timed step" if graph is not None
                         else "one Python API call per timed step")
        if shard:
            cfg["parallelism"] = (f"shard over {'batch' if shard[0].axis == 0 else 'heads'} on {world} rank(s) "
                                  "+ NCCL all-gather of O and LSE (inside each step)")
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "strong" if shard else "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic", "config": cfg,
            "pct_of_peak": 100.0 * value / world / peak,
            "roofline": ({"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                          "frac": achieved / peak, "traffic": traffic,
                          "peak_source": f"{peak_src} bf16 burst (MEASURED_PEAKS.json bf16_tflops)",
                          "frac_of_sustained_peak": achieved / peak_sus,
                          "algorithmic_bytes": w.min_hbm_bytes,
                          "traffic_source": traffic_how}
                         if intensity >= ridge else
                         {"bound": "hbm", "achieved": w.min_hbm_bytes / (avg_launch_ms * 1e-3) / 1e9,
                          "peak": measured_hbm(), "unit": "GB/s",
                          "frac": w.min_hbm_bytes / (avg_launch_ms * 1e-3) / 1e9 / measured_hbm(),
                          "traffic": traffic, "algorithmic_bytes": w.min_hbm_bytes,
                          "peak_source": "measured copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                          "arithmetic_intensity_flop_per_byte": intensity,
                          "note": "per-step time covers the attention kernel and the split merge kernel"}),
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps, "ms_per_step": e2e_ms / e2e_steps,
                    "pcie_gbs": (h2d + d2h) * e2e_steps / (e2e_ms * 1e-3) / 1e9,
                    "overlap": "two buffer sets; host->device copies, kernels and device->host copies on three "
                               "streams"},
            "clocks": clocks.summary(),
            "gpu_launches": args.steps * kernels_per_step,
            "kernel_source_hash": kernel_source_hash(),
        }
        if world == 1 and not args.no_cpu_baseline:
            from tests.parity import metrics, passes

            rows, o_ref, lse_ref, dt, threads = oracle_row_sample(w, q, k, v, args.cpu_seconds)
            if shard:
                o_all, l_all = shard[0].assemble()
            else:
                o_all, l_all = slots[0]["o"], slots[0]["lse"]
            o_gpu = o_all.cpu().to(torch.float64).numpy()
            l_gpu = l_all.cpu().to(torch.float64).numpy()
            m = metrics(o_gpu[rows[:, 0], rows[:, 2], rows[:, 1]], l_gpu[rows[:, 0], rows[:, 1], rows[:, 2]],
                        o_ref, lse_ref)
            line["cpu_baseline"] = {
                "value": row_flops(w, rows) / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                "sample": f"{len(rows)} random (b,h,i) rows of the same inputs, fp64, {dt:.1f} s"}
            line["parity"] = dict(m, rows=int(len(rows)), passes=passes(m))
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
