"""The attention kernel's static schedule, enumerated on the host by the same
iterator code the kernel runs (zyfa_attn_schedule; no GPU needed): every unit
once, heaviest query tiles first inside an L2 group, per-CTA work balanced,
and the variable-length schedule equal to the fixed-length one when all
lengths agree."""
import random

import pytest

from bf16_causal_prefill_fp8_b200 import build, zyfa

FP8, BF16 = zyfa.FP8_E4M3, zyfa.BF16
GROUP_BYTES = 48 * 1024 * 1024


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    zyfa.lib()


def all_units(grid, **kw):
    return [zyfa.attn_schedule(cta=c, grid=grid, **kw) for c in range(grid)]


def expected_units(lens, Hq):
    return sorted((b, hq, qt) for b, n in enumerate(lens) for hq in range(Hq) for qt in range((n + 127) // 128))


def cu_of(lens):
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    return cu


def tiles(units):
    return sum(qt + 1 for _, _, qt in units)


@pytest.mark.parametrize("grid", [1, 5, 148])
@pytest.mark.parametrize("lens,Hq,Hkv,Dqk,dt", [
    ([300, 0, 1, 128, 129, 1000, 77], 4, 2, 128, FP8),
    ([4096, 64, 2500, 2500, 9], 8, 1, 192, BF16),
    ([0, 0, 5], 2, 2, 128, BF16),
])
def test_varlen_covers_every_unit_once(grid, lens, Hq, Hkv, Dqk, dt):
    per = all_units(grid, Hq=Hq, Hkv=Hkv, Dqk=Dqk, dtype=dt, cu_seqlens=cu_of(lens))
    got = sorted(u for cta in per for u in cta)
    assert got == expected_units(lens, Hq)


@pytest.mark.parametrize("grid", [1, 7, 148])
@pytest.mark.parametrize("B,S,Hq,Hkv,Dqk,dt", [(2, 1000, 4, 2, 128, FP8), (3, 777, 6, 3, 192, BF16),
                                               (1, 16384, 32, 8, 128, FP8),
                                               (1, 32768, 32, 32, 128, FP8),     # 6 L2 groups of 6 slots
                                               (4, 16384, 16, 16, 192, BF16)])   # 64 slots, 4 per group
def test_fixed_covers_every_unit_once_and_equals_varlen(grid, B, S, Hq, Hkv, Dqk, dt):
    fixed = all_units(grid, Hq=Hq, Hkv=Hkv, Dqk=Dqk, dtype=dt, B=B, S=S)
    assert sorted(u for cta in fixed for u in cta) == expected_units([S] * B, Hq)
    varlen = all_units(grid, Hq=Hq, Hkv=Hkv, Dqk=Dqk, dtype=dt, cu_seqlens=cu_of([S] * B))
    assert varlen == fixed   # unit for unit, CTA by CTA


def test_group_order_is_heaviest_first():
    """With one CTA the unit list is the whole issue order: groups of (sequence,
    kv head) slots within the L2 budget, longest sequences first, and query tile
    index non-increasing inside each group."""
    rng = random.Random(3)
    lens = [rng.choice([0, 1, 127, 128, 129, 700, 5000, 30000, 70000]) for _ in range(40)]
    Hq, Hkv, Dqk, el = 4, 2, 128, 1
    order = zyfa.attn_schedule(Hq=Hq, Hkv=Hkv, Dqk=Dqk, dtype=FP8, grid=1, cta=0, cu_seqlens=cu_of(lens))
    assert sorted(order) == expected_units(lens, Hq)
    seq_order = sorted(range(len(lens)), key=lambda s: -lens[s])   # stable: equal lengths by id
    slots = [(s, h) for s in seq_order for h in range(Hkv)]
    # rebuild the greedy groups and check each group's unit run
    pos, i = 0, 0
    while i < len(slots):
        j, bytes_ = i, 0
        while j < len(slots):
            sb = lens[slots[j][0]] * (Dqk + 128) * el
            if j > i and bytes_ + sb > GROUP_BYTES:
                break
            bytes_ += sb
            j += 1
        group = set(slots[i:j])
        n = sum(Hq // Hkv * ((lens[s] + 127) // 128) for s, _ in slots[i:j])
        run = order[pos:pos + n]
        assert all((b, hq // (Hq // Hkv)) in group for b, hq, _ in run)
        qts = [qt for _, _, qt in run]
        assert qts == sorted(qts, reverse=True)
        pos, i = pos + n, j
    assert pos == len(order)


def test_per_cta_work_is_balanced():
    """The 16K GQA workload (Hq 32, Hkv 8) on 148 CTAs: tile counts differ by
    at most 2 across CTAs."""
    t = [tiles(u) for u in all_units(148, Hq=32, Hkv=8, Dqk=128, dtype=FP8, B=1, S=16384)]
    assert sum(t) == 32 * 128 * 129 // 2
    assert max(t) - min(t) <= 2
    # the per-CTA counts an instrumented run of the kernel reported on a B200
    assert (min(t), max(t)) == (1784, 1786)


def test_varlen_mix_is_balanced():
    """A mixed-length batch (64 sequences of 1..16K rows): per-CTA tile counts
    within 1 % of the mean of each other."""
    rng = random.Random(11)
    lens = [rng.randint(1, 16384) for _ in range(64)]
    t = [tiles(u) for u in all_units(148, Hq=32, Hkv=8, Dqk=128, dtype=FP8, cu_seqlens=cu_of(lens))]
    mean = sum(t) / len(t)
    assert max(t) - min(t) <= 0.01 * mean


def test_schedule_argument_errors():
    with pytest.raises(zyfa.ZyfaError):
        zyfa.attn_schedule(Hq=3, Hkv=2, Dqk=128, dtype=FP8, grid=4, cta=0, B=1, S=128)
    with pytest.raises(zyfa.ZyfaError):
        zyfa.attn_schedule(Hq=2, Hkv=2, Dqk=128, dtype=FP8, grid=4, cta=4, B=1, S=128)
    with pytest.raises(zyfa.ZyfaError):
        zyfa.attn_schedule(Hq=2, Hkv=2, Dqk=128, dtype=FP8, grid=4, cta=0, cu_seqlens=[0, 5, 3])
    assert zyfa.attn_schedule(Hq=2, Hkv=2, Dqk=128, dtype=FP8, grid=4, cta=0, cu_seqlens=[0, 0]) == []


def test_multi_group_fixed_schedule_keeps_groups_contiguous():
    """MHA 32K FP8: 8 MiB of K/V per kv head, so groups of 6 heads (48 MiB);
    with one CTA the issue order walks the groups in slot order."""
    order = zyfa.attn_schedule(Hq=32, Hkv=32, Dqk=128, dtype=FP8, grid=1, cta=0, B=1, S=32768)
    groups = [hq // 6 for _, hq, _ in order]
    assert groups == sorted(groups)
    assert len(set(groups)) == 6
