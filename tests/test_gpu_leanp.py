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
