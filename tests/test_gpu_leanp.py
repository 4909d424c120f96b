"""Lean-P codes of the attention kernel's device functions against the CPU
emulation, byte for byte (through zyfa_leanp_codes)."""
import numpy as np
import pytest
import torch

from bf16_causal_prefill_fp8_b200 import zyfa
from oracle import oracle as orc

pytestmark = pytest.mark.gpu


def _compare(s, m, bmax, A, masked=None):
    s, m, bmax, A = (np.ascontiguousarray(a, dtype=np.float32) for a in (s, m, bmax, A))
    t = lambda a: torch.from_numpy(a).cuda()
    mk = None if masked is None else torch.from_numpy(np.ascontiguousarray(masked, np.uint8)).cuda()
    code, j = zyfa.leanp_codes(t(s), t(m), t(bmax), t(A), mk)
    torch.cuda.synchronize()
    rc, rj = orc.leanp_batch(s, m, bmax, A, masked)
    got_c, got_j = code.cpu().numpy(), j.cpu().numpy()
    bad = np.flatnonzero((got_c != rc) | (got_j != rj))
    assert bad.size == 0, (f"{bad.size} mismatches, first: s={s[bad[0]]!r} m={m[bad[0]]!r} "
                           f"bmax={bmax[bad[0]]!r} A={A[bad[0]]!r} gpu=({got_c[bad[0]]},{got_j[bad[0]]}) "
                           f"cpu=({rc[bad[0]]},{rj[bad[0]]})")


def test_leanp_random_scores():
    rng = np.random.default_rng(31)
    n = 1 << 20
    m = rng.normal(0, 50, n).astype(np.float32)
    A = np.exp(rng.uniform(np.log(1e-5), np.log(30), n)).astype(np.float32)
    bmax = np.minimum(m - np.abs(rng.normal(0, 20, n)).astype(np.float32) * 8 / A, m).astype(np.float32)
    s = np.minimum(bmax - np.abs(rng.normal(0, 30, n)).astype(np.float32) / A, bmax).astype(np.float32)
    _compare(s, m, bmax, A)


def test_leanp_dense_grid_and_edges():
    A = np.float32(0.1375)
    m = np.float32(11.0)
    s = np.linspace(-2000, 11.0, 200001).astype(np.float32)
    n = s.size
    _compare(s, np.full(n, m), np.full(n, m), np.full(n, A))
    # scores landing exactly on integers of u, the block max itself, -inf, masked
    u_int = (np.arange(-50, 121, dtype=np.float32) - np.float32(120.0)) / A + m
    edge_s = np.concatenate([u_int, [m, m, -np.inf, -1e30, -3.4e38, 0.0]]).astype(np.float32)
    k = edge_s.size
    edge_s = np.minimum(edge_s, m)
    _compare(edge_s, np.full(k, m), np.full(k, m), np.full(k, A))
    masked = np.zeros(k, np.uint8); masked[::3] = 1
    _compare(edge_s, np.full(k, m), np.full(k, m), np.full(k, A), masked)


def test_leanp_block_shift_cap_and_empty_block():
    n = 4096
    rng = np.random.default_rng(32)
    m = rng.normal(0, 1e3, n).astype(np.float32)
    A = np.full(n, 3.0, np.float32)
    bmax = (m - rng.uniform(0, 2e3, n).astype(np.float32)).astype(np.float32)   # gaps past the cap
    s = bmax.copy()
    _compare(s, m, bmax, A)
    bmax_inf = np.full(n, -np.inf, np.float32)
    _compare(np.full(n, -np.inf, np.float32), m, bmax_inf, A)


def _deferred_case(rng, n, jt):
    """Scores of blocks whose shift is jt: (m - bmax) A / 8 in [jt - 8 + 1/16, jt - 7 - 1/16].
    jt < 8 puts the block max above the reference m (the deferred reference max)."""
    m = rng.normal(0, 50, n).astype(np.float32)
    A = np.exp(rng.uniform(np.log(1e-4), np.log(30), n)).astype(np.float32)
    e = (8.0 * (jt - 8) + rng.uniform(0.5, 7.5, n)).astype(np.float32)   # (m - bmax) A
    bmax = (m - e / A).astype(np.float32)
    s = (bmax - np.abs(rng.normal(0, 40, n)).astype(np.float32) / A).astype(np.float32)
    s[::17] = bmax[::17]                       # the block max itself
    return s, m, bmax, A


def test_leanp_deferred_reference_max_every_shift():
    # every block shift j the kernel can produce, -56..126: byte-exact codes
    # and shifts, the deferred regime (block max up to 64 binades above m,
    # j = -56..7) included
    rng = np.random.default_rng(33)
    parts = [_deferred_case(rng, 2048, jt) for jt in range(-56, 126)]
    s, m, bmax, A = (np.concatenate([p[i] for p in parts]) for i in range(4))
    # the cap: blocks 118 or more binades under m
    capm = rng.normal(0, 10, 4096).astype(np.float32)
    capA = np.full(4096, 2.0, np.float32)
    capb = (capm - rng.uniform(118.5 * 8 / 2.0, 2000, 4096).astype(np.float32)).astype(np.float32)
    s = np.concatenate([s, capb]); m = np.concatenate([m, capm])
    bmax = np.concatenate([bmax, capb]); A = np.concatenate([A, capA])
    _compare(s, m, bmax, A)
    _, j = orc.leanp_batch(s, m, bmax, A)
    assert set(range(-56, 127)) <= set(j.tolist())


@pytest.mark.parametrize("binades", [8, 64])
def test_leanp_deferred_limit_exact(binades):
    # (m - bmax) A = -8 binades exactly (64 binades above m is the most the
    # kernel defers): j = 8 - binades and the block max is code 120; just
    # past it j is one lower (for 64 binades the kernel moves the reference
    # before that happens; the functions still agree)
    n = 2048
    A = np.full(n, 1.0, np.float32)
    m = np.full(n, 10.0, np.float32)
    top = np.float32(10.0 + 8.0 * binades)
    bmax = np.full(n, top, np.float32)
    s = np.linspace(top - 134.0, top, n).astype(np.float32)
    _compare(s, m, bmax, A)
    code, j = orc.leanp_batch(s, m, bmax, A)
    assert np.all(j == 8 - binades) and code[-1] == 120
    bmax2 = np.full(n, top + np.float32(0.5), np.float32)
    s2 = np.minimum(s, bmax2)
    _compare(s2, m, bmax2, A)
    _, j2 = orc.leanp_batch(s2, m, bmax2, A)
    assert np.all(j2 == 7 - binades)
    # powers of two of A and m: every code 0..120 reached exactly on its integer
    u = np.arange(0, 121, dtype=np.float32)
    s3 = (u - np.float32(120.0) + top).astype(np.float32)
    k = s3.size
    c3, _ = orc.leanp_batch(s3, np.full(k, 10.0, np.float32), np.full(k, top, np.float32), np.ones(k, np.float32))
    assert np.array_equal(c3, u.astype(np.uint8))
    _compare(s3, np.full(k, 10.0, np.float32), np.full(k, top, np.float32), np.ones(k, np.float32))
