"""Host-side sharding for several GPUs (one process per GPU).

The attention forward pass splits into independent problems, one per
(batch, kv head) slot with its Hq/Hkv query heads, so ranks share nothing on
the data path: each rank runs the unchanged kernel on its own slice and no
collective is needed.  With weak scaling every rank holds a full per-GPU
workload of its own (a batch shard of the global batch).  The only
cross-rank operation is reducing timings (max over ranks), outside the timed
work.
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


def rank_seed(seed: int, rank: int) -> int:
    """Seed of a rank's own synthetic shard."""
    return seed + 1000 * rank


def max_over_ranks(x: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
