"""Multi-rank host logic on CPU: world size 2 with the gloo backend."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bf16_causal_prefill_fp8_b200 import shard


def test_partitions_cover_every_slot_once():
    for B, Hkv, world in [(1, 8, 2), (3, 5, 4), (2, 1, 3), (64, 32, 8)]:
        seen = []
        for r in range(world):
            seen += shard.slot_shard(B, Hkv, world, r)
        assert sorted(seen) == [(b, h) for b in range(B) for h in range(Hkv)]
        sizes = [shard.batch_shard(B * Hkv, world, r)[1] for r in range(world)]
        assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard.batch_shard(4, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = 10.0 + rank * 2.5
        mx = shard.max_over_ranks(local)
        seeds = shard.rank_seed(7, rank)
        slots = shard.slot_shard(1, 8, world, rank)
        dist.barrier()
        q.put((rank, mx, seeds, slots))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_disjoint_shards_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [12.5, 12.5]             # max over ranks seen by both
    assert res[0][2] != res[1][2]                           # independent seeds per rank
    assert sorted(res[0][3] + res[1][3]) == [(0, h) for h in range(8)]
    assert not set(res[0][3]) & set(res[1][3])
    assert shard.max_over_ranks(3.0) == 3.0                 # no process group: identity
