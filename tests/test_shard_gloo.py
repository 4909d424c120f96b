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
        slots = shard.slot_shard(1, 8, world, rank)
        dist.barrier()
        q.put((rank, mx, slots))
    finally:
        dist.destroy_process_group()


# one global problem: B 2, S 200, Hq 4, Hkv 2 (two query heads per kv head),
# outlier-channel K; 4 (batch, kv head) slots
PROB = dict(B=2, S=200, Hq=4, Hkv=2, Dqk=128, Dv=128, kind="outlier_k")


def _slice_outputs(rank, world):
    """The rank's share of the global problem through the oracle: its slots'
    inputs, quantized per (batch, head), fp64 attention on the dequantized
    codes and the FP8 replay.  Returns [(b, h0, h1, o_ref, o_replay)]."""
    import numpy as np
    from bf16_causal_prefill_fp8_b200 import synth
    from oracle import oracle as orc
    P = PROB
    g = P["Hq"] // P["Hkv"]
    q, k, v = synth.make_qkv(11, P["B"], P["S"], P["Hq"], P["Hkv"], P["Dqk"], P["Dv"], P["kind"])
    out = []
    for b, h0, h1 in shard.rank_slices(P["B"], P["Hkv"], world, rank):
        qs, ks, vs = shard.take(q, b, h0, h1, g), shard.take(k, b, h0, h1), shard.take(v, b, h0, h1)
        codes = [orc.quantize(x) for x in (qs, ks, vs)]
        deq = [orc.dequantize(c, sc) for c, sc in codes]
        (qc, qsc), (kc, ksc), (vc, vsc) = codes
        out.append((b, h0, h1, orc.attention(*deq),
                    orc.fp8_model(qc, kc, vc, qsc, ksc, vsc, rescale_log2=64.0)))
    return out


def _partition_worker(rank, world, port, q):
    import pickle
    import numpy as np
    # two ranks share this machine's cores: the oracle's loops get a share each
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), OMP_NUM_THREADS="2")
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = pickle.dumps(_slice_outputs(rank, world))
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        if rank == 0:
            P = PROB
            g = P["Hq"] // P["Hkv"]
            o_ref = np.full((P["B"], P["S"], P["Hq"], P["Dv"]), np.nan)
            o_rep = o_ref.copy()
            for blob in gathered:
                for b, h0, h1, a, r in pickle.loads(blob):
                    shard.put(o_ref, a, b, h0, h1, g)
                    shard.put(o_rep, r, b, h0, h1, g)
            q.put((o_ref, o_rep))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_partitioned_problem_reassembles_to_one_process_result_world2():
    # world 2 over 4 slots: every rank takes a run of (batch, kv head) slots;
    # the slices computed apart, gathered and put back, equal the whole
    # problem computed in one process (the oracle is exact per row and head,
    # and the per-(batch, head) scales do not depend on the other heads)
    import numpy as np
    from bf16_causal_prefill_fp8_b200 import synth
    from oracle import oracle as orc
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_partition_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got_ref, got_rep = q.get(timeout=120)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    P = PROB
    qf, kf, vf = synth.make_qkv(11, P["B"], P["S"], P["Hq"], P["Hkv"], P["Dqk"], P["Dv"], P["kind"])
    codes = [orc.quantize(x) for x in (qf, kf, vf)]
    (qc, qsc), (kc, ksc), (vc, vsc) = codes
    want_ref = orc.attention(*[orc.dequantize(c, sc) for c, sc in codes])
    want_rep = orc.fp8_model(qc, kc, vc, qsc, ksc, vsc, rescale_log2=64.0)
    assert not np.isnan(got_ref).any()
    assert np.array_equal(got_ref, want_ref)
    assert np.array_equal(got_rep, want_rep)


def test_rank_slices_and_take_put_round_trip():
    import numpy as np
    for B, Hkv, world in [(2, 2, 2), (1, 8, 3), (3, 5, 4), (4, 1, 3)]:
        runs = [run for r in range(world) for run in shard.rank_slices(B, Hkv, world, r)]
        covered = sorted((b, h) for b, h0, h1 in runs for h in range(h0, h1))
        assert covered == [(b, h) for b in range(B) for h in range(Hkv)]
        x = np.arange(B * 3 * Hkv * 2 * 4, dtype=np.float64).reshape(B, 3, Hkv * 2, 4)
        y = np.zeros_like(x)
        for b, h0, h1 in runs:
            part = shard.take(x, b, h0, h1, 2)
            assert part.flags["C_CONTIGUOUS"] and part.shape == (1, 3, (h1 - h0) * 2, 4)
            shard.put(y, part, b, h0, h1, 2)
        assert np.array_equal(x, y)


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
    assert sorted(res[0][2] + res[1][2]) == [(0, h) for h in range(8)]
    assert not set(res[0][2]) & set(res[1][2])
    assert shard.max_over_ranks(3.0) == 3.0                 # no process group: identity
