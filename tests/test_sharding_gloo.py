"""Multi-process (world size 2, gloo, CPU) check of the sharded forward's
orchestration, ``ForwardSharding`` (the code ``bench.py --shard`` runs over
NCCL): each rank computes its shard of one forward (the fp64 oracle stands in
for the GPU kernel here), one all-gather per tensor assembles O and LSE on
every rank, and the result equals the unsharded computation bit for bit; the
timing reduction bench.py uses (MAX over ranks) is checked on the same group."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_attention_151_b200.sharding import ForwardSharding, shard_axis, shard_bounds


def test_shard_bounds_cover_exactly_once():
    for n in range(0, 23):
        for world in range(1, 6):
            seen = []
            for r in range(world):
                a, b = shard_bounds(n, world, r)
                seen.extend(range(a, b))
                assert b - a in (n // world, n // world + 1)
            assert seen == list(range(n))


def test_axis_choice():
    assert shard_axis(8, 8) == 0 and shard_axis(4, 8) == 2 and shard_axis(1, 2) == 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _oracle_compute(scale, causal):
    import oracle
    from exact_attention_151_b200.inputs import bits

    def compute(qs, ks, vs):
        o, lse = oracle.attention(bits(qs), bits(ks), bits(vs), scale, causal, "bf16", nthreads=1)
        return torch.from_numpy(o), torch.from_numpy(lse)

    return compute


def _worker(rank, world, port, B, H, result_path):
    import oracle
    from exact_attention_151_b200.inputs import Workload, bits, make_qkv

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = Workload("shard", B=B, N=96, H=H, D=16, causal=True, seed=17)
        q, k, v = make_qkv(w)
        sh = ForwardSharding(B, w.N, H, w.D, world, rank, "cpu", torch.float64, lse_dtype=torch.float64)
        o_all, l_all = sh.run(q, k, v, _oracle_compute(w.softmax_scale, True))
        # every rank holds the whole result
        o_ref, l_ref = oracle.attention(bits(q), bits(k), bits(v), w.softmax_scale, True, "bf16", nthreads=1)
        ok = np.array_equal(o_all.numpy(), o_ref) and np.array_equal(l_all.numpy(), l_ref)
        flags = torch.tensor([1.0 if ok else 0.0], dtype=torch.float64)
        dist.all_reduce(flags, op=dist.ReduceOp.MIN)
        t = torch.tensor([float(rank + 1)], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        if rank == 0:
            with open(result_path, "w") as f:
                f.write("ok" if flags.item() == 1.0 and t.item() == float(world) else "mismatch")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("B,H", [(3, 4), (2, 4), (1, 4), (1, 3)])  # batch uneven/even, heads even/uneven
def test_two_rank_shards_reassemble_exactly(tmp_path, B, H):
    world = 2
    out = tmp_path / "result.txt"
    mp.spawn(_worker, args=(world, _free_port(), B, H, str(out)), nprocs=world, join=True)
    assert out.read_text() == "ok"


def test_single_rank_is_identity():
    import oracle
    from exact_attention_151_b200.inputs import Workload, bits, make_qkv

    w = Workload("shard1", B=2, N=40, H=2, D=16, seed=5)
    q, k, v = make_qkv(w)
    sh = ForwardSharding(2, 40, 2, 16, 1, 0, "cpu", torch.float64, lse_dtype=torch.float64)
    o, lse = sh.run(q, k, v, _oracle_compute(w.softmax_scale, False))
    o_ref, l_ref = oracle.attention(bits(q), bits(k), bits(v), w.softmax_scale, False, "bf16", nthreads=1)
    assert np.array_equal(o.numpy(), o_ref) and np.array_equal(lse.numpy(), l_ref)
