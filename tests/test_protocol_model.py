"""The attention kernel's barrier protocol, checked on a randomized model
(tests/protocol_model.py) for the kernel's three ring / buffer
configurations, and the model's power to catch planted mistakes."""
import random

import pytest

from protocol_model import BF16_D128, BF16_D192, FP8, WIDE, ProtocolError, random_units, run, run_wide

CONFIGS = {"fp8": FP8, "bf16_d128": BF16_D128, "bf16_d192": BF16_D192}


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_protocol_holds_on_random_schedules(name):
    cfg = CONFIGS[name]
    for seed in range(80):
        rng = random.Random(seed)
        run(random_units(rng), cfg, seed, p_rescale=(0.0, 0.3, 0.9)[seed % 3])


@pytest.mark.parametrize("mutation,cfg", [("pe_wait_two_back", FP8), ("no_sc_wait", FP8),
                                          ("no_sc_wait", BF16_D128), ("no_rescale_wait", FP8),
                                          ("no_rescale_wait", BF16_D128)])
def test_model_catches_planted_mistakes(mutation, cfg):
    with pytest.raises(ProtocolError):
        for seed in range(200):
            rng = random.Random(seed)
            run(random_units(rng), cfg, seed, mutation=mutation)


@pytest.mark.parametrize("mutation", ["q_slot_freed_before_copy", "mx_after_sf"])
def test_model_catches_planted_mistakes_with_q_in_tmem(mutation):
    """BF16 Dqk 128 (one S buffer, Q copied into TMEM per unit): releasing the
    Q slot before the copy has read it, and waiting for S before the other
    group's max of the previous tile (a wait two phases behind), must fail."""
    assert BF16_D128.one_s
    with pytest.raises(ProtocolError):
        for seed in range(300):
            rng = random.Random(seed)
            run(random_units(rng), BF16_D128, seed, mutation=mutation)


def test_model_catches_a_short_hand_over_ring():
    # the unit hand-over ring needs more slots than units a softmax group can
    # run ahead of the epilogue; with 2 the model finds the overwrite
    import dataclasses
    with pytest.raises(ProtocolError):
        for seed in range(400):
            rng = random.Random(seed)
            run(random_units(rng), dataclasses.replace(FP8, hand=2), seed)


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_two_producer_variant_protocol_holds(name):
    # separate K and V producer warps, each walking the tiles on its own: the
    # barrier protocol itself admits it (no aliasing, no stuck wait, no early
    # overwrite, no deadlock)
    cfg = CONFIGS[name]
    for seed in range(80):
        rng = random.Random(seed)
        run(random_units(rng), cfg, seed, p_rescale=(0.0, 0.3, 0.9)[seed % 3], two_producers=True)


def test_wide_tile_protocol_holds_on_random_schedules():
    # the FP8 kernel with 256-key tiles: one S and one P buffer shared by both
    # softmax groups, the tile max exchanged under one barrier
    for seed in range(120):
        rng = random.Random(seed)
        run_wide(random_units(rng), WIDE, seed, p_rescale=(0.0, 0.3, 0.9)[seed % 3])


@pytest.mark.parametrize("mutation", ["no_sc_wait", "no_mx_wait", "no_pe_wait", "early_sf_two_ahead"])
def test_wide_model_catches_planted_mistakes(mutation):
    with pytest.raises(ProtocolError):
        for seed in range(200):
            rng = random.Random(seed)
            run_wide(random_units(rng), WIDE, seed, mutation=mutation)


def test_wide_model_catches_a_short_hand_over_ring():
    import dataclasses
    with pytest.raises(ProtocolError):
        for seed in range(400):
            rng = random.Random(seed)
            run_wide(random_units(rng), dataclasses.replace(WIDE, hand=1), seed)
