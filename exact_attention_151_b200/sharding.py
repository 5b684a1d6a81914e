"""Host-side sharding of one attention forward across ranks (no collective on the data path).

Every (batch, head) pair is an independent problem, so a forward splits across
ranks without any exchange: contiguous batch slices when B >= world size,
otherwise contiguous head slices (copied to contiguous buffers, since a head
slice of [B, N, H, D] is strided). Each rank runs fa_fwd on its shard; if one
rank needs the whole O and LSE, a single all-gather assembles them.
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
