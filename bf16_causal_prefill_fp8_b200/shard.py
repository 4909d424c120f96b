"""Host-side sharding for several GPUs (one process per GPU).

The attention forward pass splits into independent problems, one per
(batch, kv head) slot with its Hq/Hkv query heads, so ranks share nothing on
the data path: one global problem is partitioned into contiguous runs of
slots, each rank runs the unchanged kernel on its own slice, and the slices'
outputs reassemble to the one-GPU result.  With weak scaling the global batch
grows with the number of ranks, so every rank holds a fixed per-GPU share.
The only cross-rank operation is reducing timings (max over ranks), outside
the timed work.
"""
import torch
import torch.distributed as dist


def batch_shard(global_batch: int, world: int, rank: int):
    """Contiguous batch range [start, start + count) of `rank` (sizes differ by at most one)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(global_batch, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def slot_shard(B: int, Hkv: int, world: int, rank: int):
    """The (batch, kv head) slots owned by `rank`: a contiguous run of the
    flattened slot index b * Hkv + h_kv."""
    start, count = batch_shard(B * Hkv, world, rank)
    return [(s // Hkv, s % Hkv) for s in range(start, start + count)]


def rank_slices(B: int, Hkv: int, world: int, rank: int):
    """The rank's slots as runs inside one batch entry: [(b, h0, h1)], kv heads
    h0 .. h1-1 of batch entry b (with their query heads)."""
    out = []
    for b, h in slot_shard(B, Hkv, world, rank):
        if out and out[-1][0] == b and out[-1][2] == h:
            out[-1] = (b, out[-1][1], h + 1)
        else:
            out.append((b, h, h + 1))
    return out


def take(x, b: int, h0: int, h1: int, per_slot: int = 1):
    """Contiguous copy of batch entry b, heads h0*per_slot .. h1*per_slot-1, of a
    [B, S, H, D] array or tensor (per_slot = Hq / Hkv for the query heads)."""
    part = x[b:b + 1, :, h0 * per_slot:h1 * per_slot, :]
    return part.contiguous() if hasattr(part, "contiguous") else part.copy()


def put(out, part, b: int, h0: int, h1: int, per_slot: int = 1):
    """Write a slice computed by take()'s layout back into the global [B, S, H, D] output."""
    out[b:b + 1, :, h0 * per_slot:h1 * per_slot, :] = part


def max_over_ranks(x: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
