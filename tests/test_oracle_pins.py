"""Pins of the CPU oracle against facts fixed outside of it (no GPU needed).

Each test checks one oracle function against the pages, the number format's
definition, a closed form, an invariant or an independent library routine, so
that a dropped term, a wrong sign or index or a transposed operand in the
oracle fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch

from bf16_causal_prefill_fp8_b200 import synth
from oracle import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --- e4m3 codec ----------------------------------------------------------------

def test_e4m3_decode_matches_torch_for_all_256_codes():
    ours = orc.e4m3_values()
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    nan_ours, nan_ref = np.isnan(ours), np.isnan(ref)
    assert np.array_equal(nan_ours, nan_ref)
    assert np.flatnonzero(nan_ours).tolist() == [0x7F, 0xFF]
    assert np.array_equal(ours[~nan_ours], ref[~nan_ref])
    assert ours[0x7E] == 448.0 and ours[0x08] == 2.0 ** -6 and ours[0x01] == 2.0 ** -9


def test_e4m3_power_of_two_ladder_golden():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "e4m3_pow2_ladder.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) == 15
    for k, val, code in rows:
        k, val, code = int(k), float(val), int(code)
        assert val == 2.0 ** k
        assert code == 8 * k + 56
        assert orc.e4m3_value(code) == val
        assert int(orc.e4m3_from_f32(val)[0]) == code


def test_e4m3_encode_matches_torch_rne_in_range():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(4000) * 40,
        rng.standard_normal(2000) * 0.01,                       # subnormal range
        rng.uniform(-448, 448, 2000),
        np.array([0.0, -0.0, 448.0, -448.0, 2.0 ** -10, 3 * 2.0 ** -11, 1.0625, 1.1875]),
    ]).astype(np.float32)
    ours = orc.e4m3_from_f32(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_ties_go_to_even_and_saturate():
    vals = orc.e4m3_values()
    # midpoints between consecutive positive finite codes: tie -> the even code
    for c in range(0, 0x7E):
        mid = np.float32((vals[c] + vals[c + 1]) / 2)
        if float(mid) != (vals[c] + vals[c + 1]) / 2:
            continue
        want = c if c % 2 == 0 else c + 1
        assert int(orc.e4m3_from_f32(mid)[0]) == want, c
    assert int(orc.e4m3_from_f32(1e9)[0]) == 0x7E
    assert int(orc.e4m3_from_f32(-500.0)[0]) == 0xFE
    assert int(orc.e4m3_from_f32(449.0)[0]) == 0x7E
    # round trip of every finite code
    for c in list(range(0, 0x7F)) + list(range(0x80, 0xFF)):
        assert int(orc.e4m3_from_f32(np.float32(vals[c]))[0]) == c


# --- Hadamard -----------------------------------------------------------------

def test_fwht_equals_scipy_sylvester_hadamard():
    H = scipy.linalg.hadamard(128).astype(np.float64) / math.sqrt(128.0)
    rows = orc.fwht128(np.eye(128, dtype=np.float32))
    assert np.allclose(rows, H, atol=1e-7, rtol=0)
    # orthonormal: H H^T = I
    Hf = rows.astype(np.float64)
    assert np.allclose(Hf @ Hf.T, np.eye(128), atol=1e-6)
    # applied to data it equals x @ H (H symmetric)
    x = synth.gaussian(3, 1, (7, 128))
    assert np.allclose(orc.fwht128(x), x.astype(np.float64) @ H, atol=1e-5)


def test_rotation_leaves_qk_invariant_fp64():
    q = synth.gaussian(4, 1, (16, 128)).astype(np.float64)
    k = synth.gaussian(4, 2, (16, 128)).astype(np.float64)
    H = orc.fwht128(np.eye(128, dtype=np.float32)).astype(np.float64)
    H = H / np.sqrt(np.sum(H * H, axis=1, keepdims=True))  # exact orthonormal rows
    assert np.allclose((q @ H) @ (k @ H).T, q @ k.T, atol=1e-9)


# --- quantizer ------------------------------------------------------------------

@pytest.mark.parametrize("hadamard", [False, True])
def test_quantize_scale_and_codes_properties(hadamard):
    x = synth.gaussian(5, 1, (2, 200, 3, 128))
    x[1, :, 2, :] = 0.0                                   # a zero head: scale 1, codes 0
    codes, scale = orc.quantize(x, hadamard=hadamard)
    vals = orc.e4m3_values()[codes]
    xr = orc.fwht128(x) if hadamard else x.astype(np.float32)
    for b in range(2):
        for h in range(3):
            blk = xr[b, :, h, :]
            amax = np.float32(np.max(np.abs(blk)))
            if amax == 0:
                assert scale[b, h] == 1.0 and np.all(codes[b, :, h, :] % 128 == 0)
                continue
            # the largest element lands exactly on the largest finite code
            assert np.float32(amax / np.float32(scale[b, h])) == np.float32(448.0) or \
                abs(amax / scale[b, h] - 448.0) < 1e-3
            assert np.max(np.abs(vals[b, :, h, :])) == 448.0
            # every code is the nearest e4m3 value to x/scale (brute force over codes)
            y = (blk / np.float32(scale[b, h])).astype(np.float32).astype(np.float64)
            fin = orc.e4m3_values()[:0x7F]
            d = np.abs(np.abs(y)[..., None] - fin[None, None, :])
            best = d.min(axis=-1)
            got = np.abs(vals[b, :, h, :] - np.abs(y) * 0) - 0  # decoded magnitudes
            assert np.all(np.abs(np.abs(got) - np.abs(y)) <= best + 1e-12)
            assert np.all(np.sign(vals[b, :, h, :]) * np.sign(y) >= 0)


def test_hadamard_quantize_round_trip_within_e4m3_bound():
    # rotating the dequantized codes back recovers x within e4m3's relative
    # precision (3 mantissa bits: half an ulp is 2^-4 of the value); the
    # pages' "roughly halves the input error" is reported, not asserted
    x = synth.gaussian(6, 2, (1, 256, 2, 128))
    std, _ = synth.outlier_channel_std(6, 2, 128)
    x = (x * std[None, None]).astype(np.float32)
    c1, s1 = orc.quantize(x, hadamard=True)
    back = orc.fwht128(orc.dequantize(c1, s1).astype(np.float32)).astype(np.float64)
    assert orc.rel_fro(back, x) < 2.0 ** -4
    c0, s0 = orc.quantize(x, hadamard=False)
    assert orc.rel_fro(orc.dequantize(c0, s0), x) < 2.0 ** -4


# --- attention (fp64 definition) ------------------------------------------------

def _sdpa_ref(q, k, v):
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    g = Hq // Hkv
    qt = torch.from_numpy(np.asarray(q, np.float64)).permute(0, 2, 1, 3)
    kt = torch.from_numpy(np.asarray(k, np.float64)).permute(0, 2, 1, 3).repeat_interleave(g, 1)
    vt = torch.from_numpy(np.asarray(v, np.float64)).permute(0, 2, 1, 3).repeat_interleave(g, 1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    return o.permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("shape", [(1, 1, 1, 1, 8, 8), (2, 7, 4, 2, 16, 8), (1, 33, 6, 3, 24, 16),
                                   (1, 130, 2, 2, 128, 128), (1, 64, 2, 1, 192, 128)])
def test_attention_matches_torch_sdpa(shape):
    B, S, Hq, Hkv, Dqk, Dv = shape
    q = synth.gaussian(7, 1, (B, S, Hq, Dqk)).astype(np.float64)
    k = synth.gaussian(7, 2, (B, S, Hkv, Dqk)).astype(np.float64)
    v = synth.gaussian(7, 3, (B, S, Hkv, Dv)).astype(np.float64)
    o = orc.attention(q, k, v)
    ref = _sdpa_ref(q, k, v)
    assert np.allclose(o, ref, atol=1e-12, rtol=1e-10)
    rows = [0, S - 1, S // 2]
    o2 = orc.attention(q, k, v, rows=rows)
    assert np.array_equal(o2, o[:, rows])


def test_attention_row0_is_v0_and_zero_q_gives_prefix_means():
    q = synth.gaussian(8, 1, (1, 50, 2, 16)).astype(np.float64)
    k = synth.gaussian(8, 2, (1, 50, 2, 16)).astype(np.float64)
    v = synth.gaussian(8, 3, (1, 50, 2, 16)).astype(np.float64)
    o = orc.attention(q, k, v)
    assert np.array_equal(o[:, 0], v[:, 0])
    o0 = orc.attention(np.zeros_like(q), k, v)
    pref = np.cumsum(v, axis=1) / np.arange(1, 51)[None, :, None, None]
    assert np.allclose(o0, pref, atol=1e-13)


def test_gqa_single_kv_head_equals_replicated_mha():
    q = synth.gaussian(9, 1, (1, 40, 4, 16)).astype(np.float64)
    k = synth.gaussian(9, 2, (1, 40, 1, 16)).astype(np.float64)
    v = synth.gaussian(9, 3, (1, 40, 1, 8)).astype(np.float64)
    a = orc.attention(q, k, v)
    b = orc.attention(q, np.repeat(k, 4, axis=2), np.repeat(v, 4, axis=2))
    assert np.allclose(a, b, atol=1e-14)


# --- Lean P ----------------------------------------------------------------------

def test_leanp_zero_scores_give_8j_plus_56():
    # s = m = 0: u = 56 + 8j exactly, so the code is 8j + 56 while that is a
    # finite e4m3 code (-7 <= j <= 8), the clamp value 126 above and 0 below
    # (u < 0: the shifts of a block far above the deferred reference)
    for A in [1e-4, 0.37, 5.0]:
        for j in range(-7, 9):
            assert orc.leanp_code(0.0, 0.0, A, j) == 8 * j + 56
        for j in [9, 20, 126]:
            assert orc.leanp_code(0.0, 0.0, A, j) == 126
        for j in [-8, -20, -56]:
            assert orc.leanp_code(0.0, 0.0, A, j) == 0
        assert orc.leanp_block_shift(0.0, 0.0, A) == 8
        assert orc.leanp_code(0.0, 0.0, A, 8) == 120
    assert orc.leanp_code(5.0, 5.0, 0.25, 8, masked=True) == 0
    assert orc.leanp_code(-np.inf, 5.0, 0.25, 8) == 0
    assert orc.leanp_block_shift(1.0, -np.inf, 0.5) == 8


def test_leanp_slope_formula_constant():
    A = orc.leanp_slope(1.0, 1.0, 128)
    assert A == np.float32(8.0 * math.log2(math.e) / math.sqrt(128.0))
    assert orc.leanp_slope(0.5, 0.25, 192) == np.float32(
        np.float32(0.125) * np.float32(8.0 * math.log2(math.e) / math.sqrt(192.0)))


def test_leanp_monotone_in_score():
    m, A = np.float32(3.0), np.float32(0.731)
    s = np.linspace(-200, 3.0, 20001).astype(np.float32)
    bmax = np.full_like(s, m)
    codes, js = orc.leanp_batch(s, np.full_like(s, m), bmax, np.full_like(s, A))
    assert np.all(np.diff(codes.astype(int)) >= 0)
    assert np.all(js == 8)


def test_leanp_weight_inside_mitchell_band():
    # decoded weight value(code) * 2^-j against exact 2^((s-m)A/8):
    # ratio in (2^-1/8, 1.0615] for normal codes (Mitchell's linear
    # approximation of log2 plus truncation of the code)
    rng = np.random.default_rng(11)
    n = 20000
    m = rng.uniform(-30, 30, n).astype(np.float32)
    A = np.exp(rng.uniform(np.log(1e-3), np.log(20), n)).astype(np.float32)
    # m - bmax in binades (units of 8/A).  Negative gaps are the deferred
    # reference max: a block up to 64 binades above the reference m (j = -56..7)
    gap = rng.uniform(-64, 100, n).astype(np.float32)
    bmax = (m - gap * np.float32(8.0) / A).astype(np.float32)
    frac = rng.uniform(0, 1, n)
    s = (bmax - frac * np.float32(40.0) / A).astype(np.float32)   # up to 5 binades under bmax
    s = np.minimum(s, bmax)
    codes, js = orc.leanp_batch(s, m, bmax, A)
    vals = orc.e4m3_values()[codes]
    exact = np.exp2((s.astype(np.float64) - m.astype(np.float64)) * A.astype(np.float64) / 8.0)
    w = vals * np.exp2(-js.astype(np.float64))
    normal = (codes >= 8) & (codes <= 126)
    assert normal.mean() > 0.9
    ratio = w[normal] / exact[normal]
    assert ratio.min() > 2.0 ** (-1.0 / 8.0) - 1e-4
    assert ratio.max() <= 1.0615 + 1e-4
    # the block max lands in the top binade: u in (112, 120], so its code is
    # in [112, 120] (one lower where the fp32 steps round across an integer)
    cmax, _ = orc.leanp_batch(bmax, m, bmax, A)
    cap = (js < 126) & (js >= -56)
    assert np.all((cmax[cap] >= 111) & (cmax[cap] <= 120))
    assert np.mean(cmax[cap] >= 112) > 0.99
    # the deferred regime (block max above m) is exercised, with every j -56..7
    above = bmax > m
    assert above.mean() > 0.2
    assert set(range(-56, 8)) <= set(js[above].tolist())
    assert np.all(js[above] <= 8)
    assert np.all((cmax[above & cap] >= 111) & (cmax[above & cap] <= 120))


def test_leanp_weight_doubles_when_the_reference_drops_one_binade():
    """Moving the reference down by exactly one binade (8/A) lowers the block
    shift j by one and leaves u, hence the code, unchanged, so the decoded
    weight value(code) * 2^-j doubles exactly: pins the sign of j in the
    weight and the row offset 56 + 8j, above and below the reference, with
    exact arithmetic (A = 1, integer scores)."""
    s = np.arange(-300, 41, dtype=np.float32)
    bmax = np.full_like(s, 40.0)
    A = np.ones_like(s)
    vals = orc.e4m3_values()
    for m0 in (96.0, 40.0, 8.0, -200.0, -472.0):   # block 7 binades below .. 64 binades above m
        c0, j0 = orc.leanp_batch(s, np.full_like(s, m0), bmax, A)
        c1, j1 = orc.leanp_batch(s, np.full_like(s, m0 - 8.0), bmax, A)
        assert np.all(j1 == j0 - 1) and np.array_equal(c0, c1)
        w0 = vals[c0] * np.exp2(-j0.astype(np.float64))
        w1 = vals[c1] * np.exp2(-j1.astype(np.float64))
        assert np.array_equal(w1, 2.0 * w0)
        assert c0[-1] == 120   # the block max on its integer lands on code 120


def test_leanp_block_shift_cap():
    assert orc.leanp_block_shift(1e6, -1e6, 1.0) == 126
    assert orc.leanp_block_shift(10.0, 2.0, 1.0) == 9        # gap 8*1 -> floor(1) = 1
    assert orc.leanp_block_shift(10.0, 2.0001, 1.0) == 8


def test_leanp_deferred_reference_max_boundaries():
    # A block whose max lies above the reference m (the deferred reference max
    # lets it be up to 8 binades, (bmax - m) A <= 64, above): j = 8 + floor of
    # a negative number, rounded toward minus infinity, not toward zero
    A = 1.0
    assert orc.leanp_block_shift(10.0, 10.0, A) == 8          # on the reference
    assert orc.leanp_block_shift(10.0, 10.5, A) == 7          # -0.0625 -> floor -1
    assert orc.leanp_block_shift(10.0, 18.0, A) == 7          # -1 exactly
    assert orc.leanp_block_shift(10.0, 18.5, A) == 6
    assert orc.leanp_block_shift(10.0, 74.0, A) == 0          # (m - bmax) A = -64: the limit
    assert orc.leanp_block_shift(10.0, 74.5, A) == -1         # past the limit (the kernel moves m first)
    for jt in range(0, 8):
        # (m - bmax) A = 8 (jt - 8) + 3: floor((...)/8) = jt - 8
        bm = np.float32(10.0 - (8 * (jt - 8) + 3))
        j = orc.leanp_block_shift(10.0, bm, A)
        assert j == jt
        # the block max lands in the top binade: u = 120 - 3 = 117
        assert orc.leanp_code(bm, 10.0, A, j) == 117
        # one binade under the block max: 8 codes lower
        assert orc.leanp_code(bm - 8.0, 10.0, A, j) == 109
    # at the limit the block max itself is code 120 with j = 0: weight 2^8 = 256
    assert orc.leanp_code(74.0, 10.0, A, 0) == 120
    assert orc.e4m3_values()[120] == 256.0


# --- model oracle ----------------------------------------------------------------

def _quantized_case(seed, B, S, Hq, Hkv, D, Dv=None):
    Dv = Dv or D
    q, k, v = synth.make_qkv(seed, B, S, Hq, Hkv, D, Dv)
    qc, qs = orc.quantize(q); kc, ks = orc.quantize(k); vc, vs = orc.quantize(v)
    return (qc, kc, vc, qs, ks, vs), (orc.dequantize(qc, qs), orc.dequantize(kc, ks),
                                      orc.dequantize(vc, vs)), (q, k, v)


@pytest.mark.parametrize("kv_tile", [128, 256])
def test_model_oracle_exact_p_equals_plain_definition(kv_tile):
    codes, deq, _ = _quantized_case(12, 1, 300, 4, 2, 128)
    qc, kc, vc, qs, ks, vs = codes
    o_model = orc.fp8_model(qc, kc, vc, qs, ks, vs, exact_p=True, kv_tile=kv_tile)
    o_ref = orc.attention(*deq)
    assert orc.rel_fro(o_model, o_ref) < 1e-6
    o_lazy = orc.fp8_model(qc, kc, vc, qs, ks, vs, exact_p=True, kv_tile=kv_tile, rescale_log2=64.0)
    assert orc.rel_fro(o_lazy, o_ref) < 1e-6


def test_model_oracle_tile_size_moves_the_reference_decision():
    """The deferred reference is decided once per KV tile, so 128- and 256-key
    tiles give different Lean-P codes (the first tile's max differs for rows
    past key 127), both within the FP8 bar.  (So does the exact running max:
    the codes depend on the max the tile is coded against, and that max
    covers the whole tile.)"""
    codes, deq, _ = _quantized_case(15, 1, 700, 2, 2, 128)
    qc, kc, vc, qs, ks, vs = codes
    ref = orc.attention(*deq)
    o128 = orc.fp8_model(qc, kc, vc, qs, ks, vs, rescale_log2=64.0, kv_tile=128)
    o256 = orc.fp8_model(qc, kc, vc, qs, ks, vs, rescale_log2=64.0, kv_tile=256)
    assert not np.array_equal(o128[:, 128:], o256[:, 128:])
    assert np.array_equal(o128[:, :128], o256[:, :128])   # rows 0..127 see one tile either way
    assert orc.rel_fro(o128, ref) < 3e-2 and orc.rel_fro(o256, ref) < 3e-2


def test_model_oracle_rejects_other_tile_sizes():
    codes, _, _ = _quantized_case(16, 1, 64, 1, 1, 128)
    with pytest.raises(ValueError):
        orc.fp8_model(*codes, kv_tile=192)


def _growing_score_case(seed, threshold=8.0, tile=128):
    """Q = 1.0 everywhere, K rows near a per-tile level, so the score of key j
    for every query is about 128 * level(tile of j), about 16.3 level binades
    (s * 8 log2(e) / sqrt(128) / 8), a little less for the tile max since K
    entries take the level or the next lower code at random.  For an
    8-binade deferral bound the tile max jumps by ~19 binades (rescaled), then
    ~4 (deferred), falls, then ~11 above the deferred reference (rescaled);
    for a 64-binade bound by ~70 binades (rescaled), then ~30 (deferred),
    falls, then ~78 above the reference (rescaled).  `tile` keys share a level
    (the KV tile of the replay under test)."""
    rng = np.random.default_rng(seed)
    vals = orc.e4m3_values()
    code_of = {float(vals[c]): c for c in range(0x00, 0x7F)}
    levels = {8.0: [0.5, 1.75, 2.0, 1.5, 2.5], 64.0: [0.5, 5.0, 7.0, 3.0, 10.0]}[threshold]
    S, D = tile * len(levels), 128
    qc = np.full((1, S, 1, D), code_of[1.0], dtype=np.uint8)
    kc = np.empty((1, S, 1, D), dtype=np.uint8)
    for t, lv in enumerate(levels):
        c = code_of[lv]
        kc[0, tile * t:tile * (t + 1), 0, :] = c - rng.integers(0, 2, size=(tile, D))  # lv or next lower
    vc = rng.integers(0x20, 0x50, size=(1, S, 1, D), dtype=np.uint8)
    vc |= (rng.integers(0, 2, size=vc.shape) << 7).astype(np.uint8)              # random signs
    one = np.ones((1, 1), dtype=np.float32)
    return qc, kc, vc, one, one, one


@pytest.mark.parametrize("r,tile", [(8.0, 128), (64.0, 128), (64.0, 256)])
def test_model_oracle_deferred_max_equals_plain_definition(r, tile):
    """With exact probabilities the deferred reference max (r binades) must give
    the plain softmax: pins the deferral rule, its alpha and that O and l are
    rescaled together, on scores that grow far beyond the fp32 exp2 range."""
    qc, kc, vc, qs, ks, vs = _growing_score_case(21, r, tile)
    deq = tuple(orc.dequantize(x, sc) for x, sc in ((qc, qs), (kc, ks), (vc, vs)))
    ref = orc.attention(*deq)
    o_lazy = orc.fp8_model(qc, kc, vc, qs, ks, vs, exact_p=True, rescale_log2=r, kv_tile=tile)
    assert orc.rel_fro(o_lazy, ref) < 1e-6
    # the deferral changes the Lean-P codes (the reference moves), not the bar
    o_exact = orc.fp8_model(qc, kc, vc, qs, ks, vs, kv_tile=tile)
    o_def = orc.fp8_model(qc, kc, vc, qs, ks, vs, rescale_log2=r, kv_tile=tile)
    assert not np.array_equal(o_exact, o_def)
    assert orc.rel_fro(o_def, ref) < 3e-2 and orc.rel_fro(o_exact, ref) < 3e-2
    # the case exercises what it is meant to: tile maxima (in binades) that jump
    # past the bound (a rescale), stay within it above the reference (deferred,
    # block shifts below 8), fall, and pass the bound again
    A8 = float(orc.leanp_slope(1.0, 1.0, 128)) / 8.0
    qv = orc.e4m3_values()[qc[0, 0, 0]].astype(np.float64)
    tmax = [float((orc.e4m3_values()[kc[0, tile * t:tile * t + tile, 0]].astype(np.float64) @ qv).max()) * A8
            for t in range(5)]
    assert tmax[1] - tmax[0] > r                     # moves the reference
    assert 0 < tmax[2] - tmax[1] <= r                # deferred: block above the reference
    assert tmax[3] < tmax[1]
    assert tmax[4] - tmax[1] > r                     # moves it again


@pytest.mark.parametrize("kv_tile", [128, 256])
def test_model_oracle_zero_q_gives_prefix_means(kv_tile):
    codes, deq, _ = _quantized_case(13, 1, 200, 2, 2, 128)
    qc, kc, vc, qs, ks, vs = codes
    qz = np.zeros_like(qc)
    o = orc.fp8_model(qz, kc, vc, qs, ks, vs, kv_tile=kv_tile)
    pref = np.cumsum(deq[2], axis=1) / np.arange(1, 201)[None, :, None, None]
    assert np.allclose(o, pref, atol=1e-12)
    assert np.array_equal(o[:, 0], deq[2][:, 0])


@pytest.mark.parametrize("kv_tile", [128, 256])
def test_model_oracle_leanp_error_against_fp64_is_within_fp8_bar(kv_tile):
    codes, deq, _ = _quantized_case(14, 1, 512, 2, 2, 128)
    qc, kc, vc, qs, ks, vs = codes
    o = orc.fp8_model(qc, kc, vc, qs, ks, vs, kv_tile=kv_tile, rescale_log2=64.0)
    ref = orc.attention(*deq)
    err = orc.rel_fro(o, ref)
    assert 1e-3 < err < 3e-2


# --- exact-P ablation codes --------------------------------------------------------

def test_exactp_code_power_of_two_ladder_and_masking():
    # s == m: exp2(j) exactly, whose e4m3 code is 8j + 56 (the format's ladder)
    A = orc.leanp_slope(np.float32(0.01), np.float32(0.02), 128)
    for j in range(0, 9):
        assert orc.exactp_code(3.0, 3.0, A, j) == 8 * j + 56
    assert orc.exactp_code(-np.inf, 0.0, A, 8) == 0
    assert orc.exactp_code(1.0, 2.0, A, 8, masked=True) == 0


def test_exactp_code_monotone_and_within_half_ulp():
    """Decoded weight / exact weight stays within e4m3's half-ulp bound for
    normal codes (2^-4 relative), and codes never decrease with s."""
    rng = np.random.default_rng(5)
    vals = orc.e4m3_values()
    A = np.float32(0.9)
    m = np.float32(50.0)
    s = np.sort(rng.uniform(-60.0, 50.0, 4000).astype(np.float32))
    prev = -1
    for si in s:
        j = 8
        c = orc.exactp_code(si, m, A, j)
        assert c >= prev
        prev = c
        exact = 2.0 ** ((float(si) - float(m)) * float(A) / 8.0 + j)
        if c >= 8:                                   # normal e4m3 codes
            assert abs(vals[c] / exact - 1.0) <= 2.0 ** -4 + 1e-9
    # Lean P on the same inputs is coarser: its worst ratio exceeds the exact-P bound
    lean = [vals[orc.leanp_code(si, m, A, 8)] / 2.0 ** ((float(si) - float(m)) * float(A) / 8.0 + 8)
            for si in s if orc.leanp_code(si, m, A, 8) >= 8]
    assert max(abs(x - 1.0) for x in lean) > 2.0 ** -4


def test_model_oracle_exactp_mode_prefix_means_and_bar():
    codes, deq, _ = _quantized_case(15, 1, 512, 2, 2, 128)
    qc, kc, vc, qs, ks, vs = codes
    qz = np.zeros_like(qc)
    o = orc.fp8_model(qz, kc, vc, qs, ks, vs, p_mode=2, rescale_log2=8.0)
    pref = np.cumsum(deq[2], axis=1) / np.arange(1, 513)[None, :, None, None]
    assert np.allclose(o, pref, atol=1e-12)           # equal weights: exact prefix means
    ref = orc.attention(*deq)
    e_exact = orc.rel_fro(orc.fp8_model(qc, kc, vc, qs, ks, vs, p_mode=2, rescale_log2=8.0), ref)
    e_lean = orc.rel_fro(orc.fp8_model(qc, kc, vc, qs, ks, vs, rescale_log2=8.0), ref)
    assert 1e-4 < e_exact < 3e-2 and e_exact < e_lean


# --- MLA rotation (H128 on the first 128 dims, H64 on the last 64) --------------------

def test_fwht64_matches_scipy_and_is_orthonormal():
    import scipy.linalg
    x = synth.gaussian(31, 1, (5, 64))
    ref = (x.astype(np.float64) @ scipy.linalg.hadamard(64).T) / 8.0
    assert np.allclose(orc.fwht64(x), ref, rtol=0, atol=1e-5)
    eye = orc.fwht64(np.eye(64, dtype=np.float32))
    assert np.allclose(eye @ eye.T, np.eye(64), atol=1e-6)


def test_quantize_192_rotation_is_block_diagonal_and_keeps_qk():
    """Dqk 192 with hadamard: dims 0..127 by H128, 128..191 by H64 (pinned
    through the codes: rotating first and quantizing without the flag gives the
    same bytes), and the rotation leaves Q K^T unchanged in fp64."""
    import scipy.linalg
    q = synth.gaussian(32, 1, (1, 40, 2, 192)) * np.float32(2.0)
    c_rot, s_rot = orc.quantize(q, hadamard=True)
    pre = np.concatenate([orc.fwht128(q[..., :128]), orc.fwht64(q[..., 128:])], axis=-1)
    c_pre, s_pre = orc.quantize(pre, hadamard=False)
    assert np.array_equal(c_rot, c_pre) and np.array_equal(s_rot.view(np.uint32), s_pre.view(np.uint32))
    H = np.zeros((192, 192))
    H[:128, :128] = scipy.linalg.hadamard(128) / np.sqrt(128.0)
    H[128:, 128:] = scipy.linalg.hadamard(64) / 8.0
    a = q[0, :, 0].astype(np.float64); b = q[0, :, 1].astype(np.float64)
    assert np.allclose((a @ H.T) @ (b @ H.T).T, a @ b.T, atol=1e-9)


# --- log-sum-exp output --------------------------------------------------------------

def test_attention_lse_closed_forms_and_torch():
    import torch
    q, k, _ = synth.make_qkv(33, 1, 150, 4, 2, 128, 128)
    lse = orc.attention_lse(q, k)
    sm = 1.0 / np.sqrt(128.0)
    # row 0 has one key: lse = its scaled score
    s00 = (q[0, 0].astype(np.float64) * k[0, 0, np.arange(4) // 2].astype(np.float64)).sum(-1) * sm
    assert np.allclose(lse[0, :, 0], s00, atol=1e-12)
    # Q = 0: every live score is 0, lse_i = ln(i + 1)
    lz = orc.attention_lse(np.zeros_like(q), k)
    assert np.allclose(lz[0], np.log(np.arange(1, 151))[None, :], atol=1e-12)
    # torch's logsumexp over the masked scores (GQA by repeat)
    qt = torch.from_numpy(q.astype(np.float64))[0].transpose(0, 1)                 # [H, S, D]
    kt = torch.from_numpy(k.astype(np.float64))[0].transpose(0, 1).repeat_interleave(2, dim=0)
    sc = qt @ kt.transpose(1, 2) * sm
    sc = sc.masked_fill(torch.triu(torch.ones(150, 150, dtype=torch.bool), 1), float("-inf"))
    assert np.allclose(lse[0], torch.logsumexp(sc, dim=-1).numpy(), atol=1e-10)


def test_model_lse_with_exact_weights_equals_definition():
    codes, deq, _ = _quantized_case(16, 1, 300, 2, 2, 128)
    qc, kc, vc, qs, ks, vs = codes
    for r in (0.0, 8.0):
        _, lse = orc.fp8_model(qc, kc, vc, qs, ks, vs, p_mode=1, rescale_log2=r, return_lse=True)
        assert np.allclose(lse, orc.attention_lse(deq[0], deq[1]), atol=1e-6)
    _, lse_lean = orc.fp8_model(qc, kc, vc, qs, ks, vs, rescale_log2=8.0, return_lse=True)
    assert np.abs(lse_lean - orc.attention_lse(deq[0], deq[1])).max() < 0.07   # Lean P weights: within ~6 %
