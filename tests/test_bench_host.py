"""Host-side pieces of bench.py and of the input recipe, on the CPU.

The metric, the configurations and the inputs the bench measures are fixed by
what they are, not by the kernels: these tests pin the workload table against
the published configurations (B, H, N, D, dtype, mask, input distributions),
the forward TFLOPS counting convention (4·B·H·N²·D, halved for causal), the
algorithmic byte count behind the HBM roofline, the oracle row sample's flop
count, the seeded input generator, and the rule that recorded DRAM traffic is
only reported for the kernel sources it was captured on.
"""

import json

import numpy as np
import pytest
import torch

import bench
from exact_attention_151_b200.inputs import WORKLOADS, make_dout, make_qkv

# (name, B, H, N, D, dtype, causal) of the published configurations: the small
# case, the Llama-7B shape, the long context (both masks), the sequence sweep at
# 32768 total tokens (both masks) and the ragged fp16 stress case.
PUBLISHED = [
    ("small_b1h2n256d64", 1, 2, 256, 64, "bf16", False),
    ("llama7b_b4h32n2048d128_causal", 4, 32, 2048, 128, "bf16", True),
    ("long_b1h32n8192d128_noncausal", 1, 32, 8192, 128, "bf16", False),
    ("long_b1h32n8192d128_causal", 1, 32, 8192, 128, "bf16", True),
    *[(f"sweep_n{n}_{'causal' if c else 'noncausal'}", 32768 // n, 16, n, 128, "bf16", c)
      for c in (False, True) for n in (1024, 4096, 16384, 32768)],
    ("stress_b2h16n4093d64_fp16_causal", 2, 16, 4093, 64, "fp16", True),
]


@pytest.mark.parametrize("name,B,H,N,D,dtype,causal", PUBLISHED, ids=[p[0] for p in PUBLISHED])
def test_workloads_are_the_published_configurations(name, B, H, N, D, dtype, causal):
    w = WORKLOADS[name]
    assert (w.B, w.H, w.N, w.D, w.dtype, w.causal) == (B, H, N, D, dtype, causal)
    assert w.n_keys == N and w.kv_heads == H  # self-attention
    assert w.softmax_scale == pytest.approx(1.0 / np.sqrt(D), rel=1e-15)


def test_sweep_holds_total_tokens_fixed():
    for n in (1024, 4096, 16384, 32768):
        for tag in ("causal", "noncausal"):
            w = WORKLOADS[f"sweep_n{n}_{tag}"]
            assert w.B * w.N == 32768


def test_default_workload_is_the_largest_single_gpu_forward():
    w = WORKLOADS[bench.DEFAULT_WORKLOAD]
    assert (w.B, w.H, w.N, w.D, w.causal) == (1, 16, 32768, 128, False)
    dense = [x for x in WORKLOADS.values() if not x.splitkv]
    assert w.flops == max(x.flops for x in dense)


def test_flops_follow_the_metric_convention():
    # 4·B·H·N²·D for the full product, halved for causal (square problems)
    assert WORKLOADS["llama7b_b4h32n2048d128_causal"].flops == 4 * 4 * 32 * 2048**2 * 128 / 2 == 137438953472
    assert WORKLOADS["sweep_n32768_noncausal"].flops == 4 * 1 * 16 * 32768**2 * 128
    assert WORKLOADS["sweep_n32768_causal"].flops == WORKLOADS["sweep_n32768_noncausal"].flops / 2
    assert WORKLOADS["stress_b2h16n4093d64_fp16_causal"].flops == 4 * 2 * 16 * 4093**2 * 64 / 2
    # cross lengths count the visible pairs of the bottom-right mask exactly
    w = WORKLOADS["decode_b1h32kv8nq1nk32768d128_splitkv"]
    assert w.flops == 4 * 1 * 32 * 32768 * 128  # the one query sees every key


def test_row_sample_flops_count_visible_keys():
    w = WORKLOADS["llama7b_b4h32n2048d128_causal"]
    N = 64
    rows = np.array([(0, 0, i) for i in range(N)])
    # causal row i sees i + 1 keys (square problem)
    assert bench.row_flops(w, rows) == 4.0 * w.D * N * (N + 1) / 2
    wn = WORKLOADS["long_b1h32n8192d128_noncausal"]
    assert bench.row_flops(wn, rows) == 4.0 * wn.D * N * wn.N


def test_algorithmic_bytes():
    # read Q, K, V once and write O once (16-bit), write LSE once (fp32)
    w = WORKLOADS["llama7b_b4h32n2048d128_causal"]
    assert w.min_hbm_bytes == 4 * 2048 * 32 * 128 * 2 * 4 + 4 * 32 * 2048 * 4 == 269484032
    d = WORKLOADS["decode_b8h32kv8nq1nk8192d128_splitkv"]
    kv = 2 * 8 * 8192 * 8 * 128 * 2
    assert d.min_hbm_bytes == kv + 2 * 8 * 1 * 32 * 128 * 2 + 8 * 32 * 1 * 4


def test_recorded_traffic_only_for_the_captured_sources(tmp_path, monkeypatch):
    path = tmp_path / "traffic.json"
    here = bench.kernel_source_hash()
    path.write_text(json.dumps({"a": {"dram_bytes_per_launch": 123, "kernel_source_hash": here, "how": "x"},
                                "b": {"dram_bytes_per_launch": 456, "kernel_source_hash": "0" * 16}}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    assert bench.recorded_traffic("a") == (123.0, "x")
    assert bench.recorded_traffic("b") == (None, None)  # captured on other sources
    assert bench.recorded_traffic("missing") == (None, None)


def test_source_hash_covers_every_kernel_file(tmp_path):
    base = bench.kernel_source_hash()
    assert len(base) == 16 and base == bench.kernel_source_hash()
    # a change to any one source changes the hash
    for i, src in enumerate(bench.KERNEL_SOURCES):
        copy = list(bench.KERNEL_SOURCES)
        alt = tmp_path / f"alt{i}"
        alt.write_bytes(open(src, "rb").read() + b"\n")
        copy[i] = str(alt)
        assert bench.kernel_source_hash(copy) != base
    assert bench.kernel_source_hash(bench.BWD_KERNEL_SOURCES) != base


def test_input_recipe_is_seeded_and_has_the_stated_distributions():
    w = WORKLOADS["stress_b2h16n4093d64_fp16_causal"].with_(N=1024)
    q, k, v = make_qkv(w)
    q2, _, _ = make_qkv(w)
    assert torch.equal(q, q2)  # same seed, same bits
    assert q.dtype == k.dtype == v.dtype == torch.float16
    assert q.shape == (2, 1024, 16, 64) and k.shape == v.shape == q.shape
    assert float(q.float().std()) == pytest.approx(4.0, rel=0.02)   # Q ~ N(0, 4^2)
    assert float(k.float().std()) == pytest.approx(1.0, rel=0.02)   # K ~ N(0, 1)
    vf = v.float()
    assert float(vf.min()) >= -1.0 and float(vf.max()) <= 1.0      # V ~ U(-1, 1)
    assert float(vf.std()) == pytest.approx(1 / np.sqrt(3), rel=0.02)
    other, _, _ = make_qkv(w, seed=1)
    assert not torch.equal(q, other)
    d = make_dout(w)
    assert d.shape == q.shape and not torch.equal(d, q) and torch.equal(d, make_dout(w))
