"""Host-side sharding of one attention forward across ranks.

Every (batch, head) pair is an independent problem (the FA2 work partition
over batch x heads x query blocks, mlqm.cn FA1/FA2 comparison, section 2.1),
so a forward splits across ranks with no exchange while it computes:
contiguous batch slices when B >= world size, otherwise contiguous head
slices (copied to contiguous buffers, since a head slice of [B, N, H, D] is
strided). Each rank runs the fused kernel on its shard; when every rank needs
the whole O and LSE, one all-gather per tensor assembles them.

``ForwardSharding`` is the orchestration ``bench.py --shard`` runs over NCCL;
the world-size-2 gloo test runs the same code on CPU with another compute
function standing in for the kernel.
"""

from __future__ import annotations


def shard_bounds(n_units: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous, balanced [start, stop) of n_units for `rank` of `world` (sizes differ by at most 1)."""
    if world < 1 or not 0 <= rank < world or n_units < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(n_units, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def shard_axis(B: int, world: int) -> int:
    """The [B, N, H, D] axis to split: batch (0) if it has a unit per rank, else heads (2)."""
    return 0 if B >= world else 2


def take_shard(t, world: int, rank: int, axis: int):
    """This rank's contiguous shard of a [B, N, H, D] (or [B, H, N] for axis mapping 0->0, 2->1) tensor."""
    start, stop = shard_bounds(t.shape[axis], world, rank)
    return t.narrow(axis, start, stop - start).contiguous()


def gather_shards(parts, axis: int):
    """Concatenate per-rank shards (in rank order) back along `axis`."""
    import torch

    return torch.cat(list(parts), dim=axis)


class ForwardSharding:
    """One [B, N, H, D] forward split over the ranks of a process group.

    ``local(t)`` is this rank's shard of an input; ``gather(o, lse)`` takes
    this rank's outputs (O shard in the input layout, LSE shard [B', H', N])
    and returns the whole O [B, N, H, D] and LSE [B, H, N] on every rank,
    through one ``all_gather_into_tensor`` per tensor. Shards that differ in
    size by one unit travel in buffers padded to the largest shard. Send and
    receive buffers are allocated once, so a timed loop reuses them.
    """

    def __init__(self, B: int, N: int, H: int, D: int, world: int, rank: int, device, dtype, group=None,
                 lse_dtype=None):
        import torch

        lse_dtype = torch.float32 if lse_dtype is None else lse_dtype
        self.B, self.N, self.H, self.D = B, N, H, D
        self.world, self.rank, self.group = world, rank, group
        self.axis = shard_axis(B, world)
        self.lse_axis = 0 if self.axis == 0 else 1
        units = B if self.axis == 0 else H
        self.bounds = [shard_bounds(units, world, r) for r in range(world)]
        self.n_max = max(b - a for a, b in self.bounds)
        self.count = self.bounds[rank][1] - self.bounds[rank][0]
        self.even = all(b - a == self.n_max for a, b in self.bounds)
        if self.axis == 0:
            o_pad, l_pad = (self.n_max, N, H, D), (self.n_max, H, N)
        else:
            o_pad, l_pad = (B, N, self.n_max, D), (B, self.n_max, N)
        self.o_pad_shape, self.l_pad_shape = o_pad, l_pad
        self.o_send = torch.zeros(o_pad, dtype=dtype, device=device)
        self.l_send = torch.zeros(l_pad, dtype=lse_dtype, device=device)
        self.o_recv = torch.empty((world,) + o_pad, dtype=dtype, device=device)
        self.l_recv = torch.empty((world,) + l_pad, dtype=lse_dtype, device=device)

    def local(self, t):
        """This rank's contiguous shard of a [B, N, H, D] tensor."""
        return take_shard(t, self.world, self.rank, self.axis)

    def local_lse_shape(self):
        shape = list(self.l_pad_shape)
        shape[self.lse_axis] = self.count
        return tuple(shape)

    def exchange(self, o, lse):
        """All-gather this rank's O and LSE shards into the receive buffers."""
        import torch.distributed as dist

        if self.even:
            o_in, l_in = o, lse
        else:
            self.o_send.narrow(self.axis, 0, self.count).copy_(o)
            self.l_send.narrow(self.lse_axis, 0, self.count).copy_(lse)
            o_in, l_in = self.o_send, self.l_send
        if self.world == 1:
            self.o_recv[0].copy_(o_in)
            self.l_recv[0].copy_(l_in)
            return
        dist.all_gather_into_tensor(self.o_recv.view(-1), o_in.reshape(-1), group=self.group)
        dist.all_gather_into_tensor(self.l_recv.view(-1), l_in.reshape(-1), group=self.group)

    def assemble(self):
        """The whole O [B, N, H, D] and LSE [B, H, N] from the receive buffers (rank order)."""
        o_parts, l_parts = [], []
        for r, (a, b) in enumerate(self.bounds):
            o_parts.append(self.o_recv[r].narrow(self.axis, 0, b - a))
            l_parts.append(self.l_recv[r].narrow(self.lse_axis, 0, b - a))
        return gather_shards(o_parts, self.axis), gather_shards(l_parts, self.lse_axis)

    def gather(self, o, lse):
        self.exchange(o, lse)
        return self.assemble()

    def run(self, q, k, v, compute):
        """Shard q, k, v, run ``compute(qs, ks, vs) -> (o_shard, lse_shard)`` and gather.

        Returns the whole (O, LSE) on every rank."""
        o, lse = compute(self.local(q), self.local(k), self.local(v))
        return self.gather(o, lse)
