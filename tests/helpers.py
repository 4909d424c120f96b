"""Shared helpers of the GPU parity tests: seeded inputs, the CUDA path through
the C-ABI binding, and the oracle's references for the same inputs."""
import numpy as np
import torch

from bf16_causal_prefill_fp8_b200 import synth, zyfa
from oracle import oracle as orc

# Tolerances (relative Frobenius error of the bf16 output against the fp64
# oracle on the values the GPU received): the acceptance bars of the method.
TOL_BF16 = 5e-3
TOL_FP8 = 3e-2
# GPU against the CPU replay of the FP8 pipeline (same codes, same tile order):
# separates kernel bugs from the method's own error.  Budget: bf16 output
# rounding (2^-9/sqrt(3) ~ 1.1e-3) plus one-step Lean-P code flips (a weight
# off by 2^(1/8)) wherever the tensor core's fp32 sum of a score differs from
# the oracle's fp64 sum near an integer boundary of u; with heavy-tailed
# outlier channels the scores are large and flips are more frequent (measured
# 4.0e-3 on the outlier-K case).  A layout or scale bug in the kernel moves
# the error to >= 1e-1, far above this budget.
TOL_FP8_MODEL = 8e-3
# The kernel's deferred reference max: it moves when a tile's max exceeds it
# by more than this many binades (the CPU replay takes the same rule).
RESCALE_LOG2 = 64.0


def bf16_round(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16)


def inputs(seed, B, S, Hq, Hkv, Dqk, Dv, kind="gaussian", q_gain=1.0):
    q, k, v = synth.make_qkv(seed, B, S, Hq, Hkv, Dqk, Dv, kind)
    if q_gain != 1.0:
        q = (q * np.float32(q_gain)).astype(np.float32)
    return q, k, v


def run_bf16(q, k, v):
    qb, kb, vb = bf16_round(q), bf16_round(k), bf16_round(v)
    o = zyfa.attn_fwd(qb.cuda(), kb.cuda(), vb.cuda())
    torch.cuda.synchronize()
    return o.float().cpu().numpy().astype(np.float64), (qb.double().numpy(), kb.double().numpy(),
                                                       vb.double().numpy())


def quantize_gpu(x: np.ndarray, hadamard=False, as_bf16=False):
    t = bf16_round(x) if as_bf16 else torch.from_numpy(np.ascontiguousarray(x))
    codes, scale = zyfa.quantize(t.cuda(), hadamard=hadamard)
    torch.cuda.synchronize()
    return codes, scale


def run_fp8(q, k, v, hadamard=False, check_prepass=True):
    """Quantize on the GPU, run FP8 attention, and return the output plus the
    oracle's own quantization (asserted bit-identical to the GPU's)."""
    qc, qs = quantize_gpu(q, hadamard)
    kc, ks = quantize_gpu(k, hadamard)
    vc, vs = quantize_gpu(v, False)
    o = zyfa.attn_fwd(qc, kc, vc, q_scale=qs, k_scale=ks, v_scale=vs)
    torch.cuda.synchronize()
    oq = orc.quantize(q, hadamard=hadamard)
    ok = orc.quantize(k, hadamard=hadamard)
    ov = orc.quantize(v, hadamard=False)
    if check_prepass:
        for (gc, gs), (rc, rs) in zip(((qc, qs), (kc, ks), (vc, vs)), (oq, ok, ov)):
            assert np.array_equal(gc.cpu().numpy(), rc)
            assert np.array_equal(gs.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    return o.float().cpu().numpy().astype(np.float64), (oq, ok, ov)


def fp8_references(codes, rows=None):
    (qc, qs), (kc, ks), (vc, vs) = codes
    deq = (orc.dequantize(qc, qs), orc.dequantize(kc, ks), orc.dequantize(vc, vs))
    ref = orc.attention(*deq, rows=rows)
    model = orc.fp8_model(qc, kc, vc, qs, ks, vs, rows=rows, rescale_log2=RESCALE_LOG2,
                          kv_tile=fp8_kv_tile(qc.shape[3]))
    return ref, model


def fp8_kv_tile(Dqk):
    """Keys per KV tile of the FP8 kernel for this Dqk, as the library reports it: the
    CPU replay takes the deferred reference-max decision at the same tiles."""
    from bf16_causal_prefill_fp8_b200 import zyfa
    return zyfa.kv_tile(zyfa.FP8_E4M3, Dqk)


# Localised bounds.  A whole-tensor relative error dilutes one bad head or one
# bad query tile; these are checked beside it.  Per head: the same bars as the
# whole tensor (every head has the same statistics).  Per (batch, row, head)
# output vector: the FP8 method's own error is not bounded per row (a weight
# off by up to one Lean-P step moves a row that averages few keys by several
# percent), so the per-row bars sit well above the method's scatter and well
# below what a corrupted tile gives (an unrelated or zeroed vector: relative
# error near 1 or above).
ROW_TOL_BF16 = 2e-2
ROW_TOL_FP8 = 1e-1
ROW_TOL_FP8_MODEL = 5e-2


def head_errors(got, ref):
    """Relative Frobenius error of each query head over (batch, rows, Dv)."""
    d = np.asarray(got, np.float64) - np.asarray(ref, np.float64)
    num = np.sqrt((d * d).sum(axis=(0, 1, 3)))
    den = np.sqrt((np.asarray(ref, np.float64) ** 2).sum(axis=(0, 1, 3)))
    return num / den


def row_errors(got, ref):
    """Relative error of each (batch, row, head) output vector over Dv."""
    d = np.asarray(got, np.float64) - np.asarray(ref, np.float64)
    num = np.sqrt((d * d).sum(axis=3))
    den = np.sqrt((np.asarray(ref, np.float64) ** 2).sum(axis=3))
    return num / np.maximum(den, 1e-300)


def check_local(got, ref, head_tol, row_tol, what, rows=None):
    """Assert the per-head and per-row bounds; returns (worst head, worst row)."""
    he, re = head_errors(got, ref), row_errors(got, ref)
    b, r, h = np.unravel_index(int(np.argmax(re)), re.shape)
    row = int(rows[r]) if rows is not None else int(r)
    print(f"{what}: worst head {he.max():.3e} (head {int(np.argmax(he))}); "
          f"worst row {re.max():.3e} (batch {b}, row {row}, head {h})")
    assert he.max() <= head_tol, (what, "head", int(np.argmax(he)), float(he.max()))
    assert re.max() <= row_tol, (what, "row", int(b), row, int(h), float(re.max()))
    return float(he.max()), float(re.max())


def tile_rows(S, seed, tile=128):
    """One seeded row inside every `tile`-row query tile, plus each tile's
    first and last row for the first and last two tiles, the middle tile and
    the ragged tail: every query tile of every head is sampled."""
    rng = np.random.default_rng(seed)
    starts = np.arange(0, S, tile)
    inner = starts + rng.integers(0, tile, size=len(starts))
    inner = np.minimum(inner, S - 1)
    edges = []
    for t0 in (0, tile, (S // 2) // tile * tile, starts[-1] - tile, starts[-1]):
        if 0 <= t0 < S:
            edges += [t0, min(t0 + tile - 1, S - 1)]
    edges += [1, S - 1]
    r = np.unique(np.concatenate([inner, edges]))
    return r[r < S].astype(np.int32)
