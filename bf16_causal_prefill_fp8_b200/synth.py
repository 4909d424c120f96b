"""Seeded synthetic Q/K/V generators (numpy, CPU).

Shared by the tests, the bench and the CPU oracle's callers.  This module holds
none of the attention method's arithmetic: it only draws inputs.

Generator: a counter-based SplitMix64 stream per (seed, stream id).  Element n
of a stream is the SplitMix64 output for counter n + 1 under the stream key;
pairs of 53-bit uniforms go through Box-Muller (fp64) to two normals, rounded
once to fp32.  Results are independent of chunking and of the machine.

Stream ids: Q = 1, K = 2, V = 3, per-channel std = 4, outlier channel picks = 5.
"""
import os

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
M1 = np.uint64(0xBF58476D1CE4E5B9)
M2 = np.uint64(0x94D049BB133111EB)
STREAM_Q, STREAM_K, STREAM_V, STREAM_CHSTD, STREAM_OUTLIER = 1, 2, 3, 4, 5

_CHUNK = 1 << 22


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * M1
    z = (z ^ (z >> np.uint64(27))) * M2
    return z ^ (z >> np.uint64(31))


def _key(seed: int, stream: int) -> np.uint64:
    with np.errstate(over="ignore"):
        z = np.array([(int(seed) * 0x9E3779B97F4A7C15 + int(stream) * 0xD1B54A32D192ED03)
                      & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64)
        return _mix(z)[0]


def uniform64(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """Uniform doubles in [0, 1) for counters start .. start+count-1 of a stream."""
    key = _key(seed, stream)
    n = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = _mix(key + n * GOLDEN)
    return (z >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def _normal_pairs(seed: int, stream: int, p0: int, p1: int) -> np.ndarray:
    """Box-Muller outputs of pairs p0 .. p1-1 of a stream (elements 2 p0 .. 2 p1 - 1)."""
    u = uniform64(seed, stream, 2 * p0, 2 * (p1 - p0))
    u1, u2 = u[0::2], u[1::2]
    r = np.sqrt(-2.0 * np.log1p(-u1))
    th = 2.0 * np.pi * u2
    z = np.empty(2 * (p1 - p0), dtype=np.float64)
    z[0::2] = r * np.cos(th)
    z[1::2] = r * np.sin(th)
    return z.astype(np.float32)


def normal_f32(seed: int, stream: int, count: int, start: int = 0) -> np.ndarray:
    """Elements start .. start+count-1 of a stream's N(0,1) draws, rounded to
    fp32 (Box-Muller on consecutive pairs; start must be even).  Large requests
    are split into chunks computed on several threads: every element depends
    on its counter only, so the values do not depend on the split."""
    if start % 2:
        raise ValueError("start must be even (draws come in Box-Muller pairs)")
    out = np.empty(count, dtype=np.float32)
    q0 = start // 2
    npairs = (count + 1) // 2
    spans = [(p0, min(npairs, p0 + _CHUNK)) for p0 in range(0, npairs, _CHUNK)]

    def fill(span):
        p0, p1 = span
        z = _normal_pairs(seed, stream, q0 + p0, q0 + p1)
        lo, hi = 2 * p0, min(count, 2 * p1)
        out[lo:hi] = z[: hi - lo]

    if len(spans) > 1:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=min(len(spans), os.cpu_count() or 1)) as ex:
            list(ex.map(fill, spans))
    else:
        for sp in spans:
            fill(sp)
    return out


def gaussian(seed: int, stream: int, shape, start: int = 0) -> np.ndarray:
    return normal_f32(seed, stream, int(np.prod(shape)), start).reshape(shape)


def outlier_channel_std(seed: int, H: int, D: int, n_outliers: int = 4, factor: float = 20.0):
    """Per-(head, channel) std: lognormal(0, 1) from stream 4, and n_outliers
    distinct channels per head (partial Fisher-Yates driven by stream 5) scaled
    by `factor`.  Returns (std fp32 [H, D], picks int [H, n_outliers])."""
    std = np.exp(normal_f32(seed, STREAM_CHSTD, H * D).astype(np.float64)).reshape(H, D)
    u = uniform64(seed, STREAM_OUTLIER, 0, H * n_outliers).reshape(H, n_outliers)
    picks = np.empty((H, n_outliers), dtype=np.int64)
    for h in range(H):
        perm = list(range(D))
        for i in range(n_outliers):
            jj = i + int(u[h, i] * (D - i))
            perm[i], perm[jj] = perm[jj], perm[i]
            picks[h, i] = perm[i]
        std[h, picks[h]] *= factor
    return std.astype(np.float32), picks


def make_qkv(seed: int, B: int, S: int, Hq: int, Hkv: int, Dqk: int, Dv: int,
             kind: str = "gaussian", b0: int = 0, nb: int = None):
    """Q [B,S,Hq,Dqk], K [B,S,Hkv,Dqk], V [B,S,Hkv,Dv] fp32; with b0 / nb only
    batch entries b0 .. b0+nb-1 of those tensors (the same values as slicing
    the whole batch: each entry's draws start at its own counter).

    kind = "gaussian": i.i.d. N(0,1).
    kind = "outlier_k": K channels scaled by outlier_channel_std (heavy-tailed,
        4 channels per kv head x20), Q and V N(0,1).
    kind = "mla": N(0,1) with Q and K dims 128 .. Dqk-1 (the rope part) x2.
    """
    nb = B - b0 if nb is None else nb
    if not (0 <= b0 and nb >= 0 and b0 + nb <= B):
        raise ValueError("batch range outside [0, B)")
    q = gaussian(seed, STREAM_Q, (nb, S, Hq, Dqk), b0 * S * Hq * Dqk)
    k = gaussian(seed, STREAM_K, (nb, S, Hkv, Dqk), b0 * S * Hkv * Dqk)
    v = gaussian(seed, STREAM_V, (nb, S, Hkv, Dv), b0 * S * Hkv * Dv)
    if kind == "outlier_k":
        std, _ = outlier_channel_std(seed, Hkv, Dqk)
        k *= std[None, None, :, :]
    elif kind == "mla":
        q[..., 128:] *= np.float32(2.0)
        k[..., 128:] *= np.float32(2.0)
    elif kind != "gaussian":
        raise ValueError(f"unknown input kind {kind!r}")
    return q, k, v


def make_qkv_rows(seed: int, T: int, Hq: int, Hkv: int, Dqk: int, Dv: int, kind: str, r0: int, r1: int):
    """Rows r0 .. r1-1 of make_qkv(seed, 1, T, ...)[i][0]: a slice of packed
    [T, H, D] tensors (each row's draws start at its own counter)."""
    if not 0 <= r0 <= r1 <= T:
        raise ValueError("row range outside [0, T)")
    n = r1 - r0
    q = gaussian(seed, STREAM_Q, (n, Hq, Dqk), r0 * Hq * Dqk)
    k = gaussian(seed, STREAM_K, (n, Hkv, Dqk), r0 * Hkv * Dqk)
    v = gaussian(seed, STREAM_V, (n, Hkv, Dv), r0 * Hkv * Dv)
    if kind == "outlier_k":
        std, _ = outlier_channel_std(seed, Hkv, Dqk)
        k *= std[None, :, :]
    elif kind == "mla":
        q[..., 128:] *= np.float32(2.0)
        k[..., 128:] *= np.float32(2.0)
    elif kind != "gaussian":
        raise ValueError(f"unknown input kind {kind!r}")
    return q, k, v


# Workloads: the sizes and input structure of the pages' benchmarks.
WORKLOADS = {
    "tiny_s512": dict(B=1, S=512, Hq=2, Hkv=2, Dqk=128, Dv=128, kind="gaussian"),
    "gqa32x8_s16k_outlier": dict(B=1, S=16384, Hq=32, Hkv=8, Dqk=128, Dv=128, kind="outlier_k"),
    "mha32_s32k": dict(B=1, S=32768, Hq=32, Hkv=32, Dqk=128, Dv=128, kind="gaussian"),
    "mla16_s16k_192_128": dict(B=1, S=16384, Hq=16, Hkv=16, Dqk=192, Dv=128, kind="mla"),
}
for _s in (1024, 2048, 4096, 8192, 16384, 32768, 65536):
    WORKLOADS[f"sweep_s{_s // 1024}k"] = dict(B=65536 // _s, S=_s, Hq=32, Hkv=32, Dqk=128,
                                             Dv=128, kind="gaussian")


# Packed (variable-length) batches: the pages measure fixed lengths only, so
# this mix is a stand-in for serving traffic: n lengths drawn log-uniform in
# [lo, hi] (stream 9), packed in draw order.
VARLEN_WORKLOADS = {
    "varlen_gqa32x8_mix32": dict(Hq=32, Hkv=8, Dqk=128, Dv=128, kind="outlier_k", nseq=32, lo=512, hi=16384),
}


def varlen_lengths(seed: int, n: int, lo: int, hi: int) -> list:
    u = uniform64(seed, 9, 0, n)
    return [int(round(lo * (hi / lo) ** float(x))) for x in u]


def causal_flops(B: int, S: int, Hq: int, Dqk: int, Dv: int) -> float:
    """FLOP count of causal attention, FlashAttention convention 2*B*Hq*(S^2/2)*(Dqk+Dv)."""
    return 2.0 * B * Hq * (S * S / 2.0) * (Dqk + Dv)
