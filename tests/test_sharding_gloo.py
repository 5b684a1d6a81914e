"""Multi-process (world size 2, gloo, CPU) check of the host-side sharding:
each rank computes its shard of one forward (the fp64 oracle stands in for the
GPU kernel here), one all-gather assembles O and LSE, and the result equals the
unsharded computation bit for bit; the timing reduction bench.py uses (MAX over
ranks) is checked on the same group."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_attention_151_b200.sharding import gather_shards, shard_axis, shard_bounds, take_shard


def test_shard_bounds_cover_exactly_once():
    for n in range(0, 23):
        for world in range(1, 6):
            seen = []
            for r in range(world):
                a, b = shard_bounds(n, world, r)
                seen.extend(range(a, b))
                assert b - a in (n // world, n // world + 1)
            assert seen == list(range(n))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, B, result_path):
    import oracle
    from exact_attention_151_b200.inputs import Workload, bits, make_qkv

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = Workload("shard", B=B, N=96, H=4, D=16, causal=True, seed=17)
        q, k, v = make_qkv(w)
        axis = shard_axis(B, world)
        qs, ks, vs = (take_shard(t, world, rank, axis) for t in (q, k, v))
        o, lse = oracle.attention(bits(qs), bits(ks), bits(vs), w.softmax_scale, True, "bf16", nthreads=1)
        o, lse = torch.from_numpy(o), torch.from_numpy(lse)
        # shards may differ in size by one unit: gather through a padded buffer
        n_max = shard_bounds(q.shape[axis], world, 0)[1]
        lse_axis = 0 if axis == 0 else 1
        pad_o = torch.zeros(o.shape[:axis] + (n_max,) + o.shape[axis + 1:], dtype=o.dtype)
        pad_o.narrow(axis, 0, o.shape[axis]).copy_(o)
        pad_l = torch.zeros(lse.shape[:lse_axis] + (n_max,) + lse.shape[lse_axis + 1:], dtype=lse.dtype)
        pad_l.narrow(lse_axis, 0, lse.shape[lse_axis]).copy_(lse)
        go = [torch.zeros_like(pad_o) for _ in range(world)]
        gl = [torch.zeros_like(pad_l) for _ in range(world)]
        dist.all_gather(go, pad_o)
        dist.all_gather(gl, pad_l)
        sizes = [shard_bounds(q.shape[axis], world, r) for r in range(world)]
        o_all = gather_shards([g.narrow(axis, 0, b - a) for g, (a, b) in zip(go, sizes)], axis)
        l_all = gather_shards([g.narrow(lse_axis, 0, b - a) for g, (a, b) in zip(gl, sizes)], lse_axis)
        t = torch.tensor([float(rank + 1)], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        if rank == 0:
            o_ref, l_ref = oracle.attention(bits(q), bits(k), bits(v), w.softmax_scale, True, "bf16", nthreads=1)
            ok = (np.array_equal(o_all.numpy(), o_ref) and np.array_equal(l_all.numpy(), l_ref)
                  and t.item() == float(world))
            with open(result_path, "w") as f:
                f.write("ok" if ok else "mismatch")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("B", [3, 1])  # batch split (uneven) and head split
def test_two_rank_shards_reassemble_exactly(tmp_path, B):
    world = 2
    out = tmp_path / "result.txt"
    mp.spawn(_worker, args=(world, _free_port(), B, str(out)), nprocs=world, join=True)
    assert out.read_text() == "ok"
