"""The localised bounds of the full-size parity tests, checked on the CPU with
planted mistakes: at 16K rows and 32 heads, one corrupted 128-row query tile
of one head (an unrelated vector, a zeroed tile, a tile scaled by 1.2) passes
the whole-tensor bound but fails the per-head or per-row one, and the row
sampler touches every query tile."""
import numpy as np
import pytest

from helpers import ROW_TOL_FP8, TOL_FP8, check_local, tile_rows
from oracle import oracle as orc

S, HQ, DV = 16384, 32, 128


def test_tile_rows_cover_every_query_tile():
    for S_ in (1, 127, 128, 129, 700, 16384, 32768, 65536):
        r = tile_rows(S_, 3)
        assert r.min() >= 0 and r.max() < S_ and np.all(np.diff(r) > 0)
        assert set(range((S_ + 127) // 128)) <= set((r // 128).tolist())
        assert S_ - 1 in r and 0 in r


@pytest.mark.parametrize("corruption", ["unrelated", "zero", "scaled"])
def test_one_corrupted_tile_of_one_head_fails(corruption):
    rng = np.random.default_rng(0)
    rows = tile_rows(S, 3)
    ref = rng.standard_normal((1, len(rows), HQ, DV))
    # the method's own scatter: 2 % relative noise on every output vector
    got = ref * (1 + 0.02 * rng.standard_normal(ref.shape))
    check_local(got, ref, TOL_FP8, ROW_TOL_FP8, "clean")
    head, tile = 5, 77
    sel = (rows // 128) == tile
    assert sel.any()
    bad = got.copy()
    if corruption == "unrelated":
        bad[:, sel, head] = rng.standard_normal(bad[:, sel, head].shape)
    elif corruption == "zero":
        bad[:, sel, head] = 0.0
    else:
        bad[:, sel, head] *= 1.2
    assert orc.rel_fro(bad, ref) <= TOL_FP8          # the whole-tensor bound alone misses it
    with pytest.raises(AssertionError):
        check_local(bad, ref, TOL_FP8, ROW_TOL_FP8, corruption)
