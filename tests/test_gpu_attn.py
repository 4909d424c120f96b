"""Causal attention through zyfa_attn_fwd against the fp64 oracle.

BF16: relative Frobenius error <= 5e-3 against fp64 attention on the bf16
inputs.  FP8: <= 3e-2 against fp64 attention on the dequantized e4m3 inputs,
and close to the CPU replay of the FP8 pipeline (same codes, same order).
Sizes span several 128-row tiles and ragged tails."""
import numpy as np
import pytest
import torch

from bf16_causal_prefill_fp8_b200 import zyfa
from oracle import oracle as orc

from helpers import (RESCALE_LOG2, ROW_TOL_BF16, ROW_TOL_FP8, ROW_TOL_FP8_MODEL, TOL_BF16, TOL_FP8, TOL_FP8_MODEL,
                     bf16_round, check_local, fp8_kv_tile, fp8_references, inputs, run_bf16, run_fp8)

pytestmark = pytest.mark.gpu

SHAPES = [  # B, S, Hq, Hkv, Dqk, Dv
    (1, 1, 1, 1, 128, 128),
    (1, 64, 2, 2, 128, 128),
    (1, 127, 2, 2, 128, 128),
    (1, 128, 2, 2, 128, 128),
    (1, 129, 2, 2, 128, 128),
    (1, 512, 2, 2, 128, 128),        # the pages' tiny configuration
    (2, 300, 4, 2, 128, 128),        # GQA, batch 2
    (1, 1000, 6, 1, 128, 128),       # GQA, one kv head
    (1, 300, 2, 2, 192, 128),        # MLA shape
    (2, 200, 4, 4, 192, 128),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_bf16_parity(shape):
    B, S, Hq, Hkv, Dqk, Dv = shape
    q, k, v = inputs(41, B, S, Hq, Hkv, Dqk, Dv, kind="mla" if Dqk == 192 else "gaussian")
    o, (qd, kd, vd) = run_bf16(q, k, v)
    ref = orc.attention(qd, kd, vd)
    err = orc.rel_fro(o, ref)
    print(f"bf16 {shape}: vs fp64 {err:.3e}")
    assert err <= TOL_BF16, err
    assert np.array_equal(o[:, 0], np.asarray(torch.from_numpy(vd[:, 0]).repeat_interleave(Hq // Hkv, 1)
                                              .to(torch.bfloat16).double()))


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_fp8_parity(shape):
    B, S, Hq, Hkv, Dqk, Dv = shape
    q, k, v = inputs(42, B, S, Hq, Hkv, Dqk, Dv, kind="mla" if Dqk == 192 else "gaussian")
    o, codes = run_fp8(q, k, v)
    ref, model = fp8_references(codes)
    err = orc.rel_fro(o, ref)
    err_model = orc.rel_fro(o, model)
    print(f"fp8 {shape}: vs fp64 {err:.3e}  vs model {err_model:.3e}")
    assert err <= TOL_FP8, err
    assert err_model <= TOL_FP8_MODEL, err_model


@pytest.mark.parametrize("S", [255, 256, 257, 383, 384, 385, 511, 513, 640, 767])
def test_fp8_kv_tile_edges(S):
    """Sequence lengths around the 256-key KV tile: the last tile of a unit
    holds the diagonal in its first half (even query tile, second half all
    masked) or in its second half (odd query tile), and the ragged tail reads
    zero-filled rows.  FP8 against fp64 and the replay with the kernel's own
    KV tile; BF16 on the same values."""
    q, k, v = inputs(51, 1, S, 4, 2, 128, 128, kind="outlier_k")
    o, codes = run_fp8(q, k, v)
    ref, model = fp8_references(codes)
    e_ref, e_model = orc.rel_fro(o, ref), orc.rel_fro(o, model)
    print(f"fp8 S={S}: vs fp64 {e_ref:.3e}  vs model {e_model:.3e}")
    assert e_ref <= TOL_FP8 and e_model <= TOL_FP8_MODEL
    check_local(o, model, TOL_FP8_MODEL, ROW_TOL_FP8_MODEL, f"fp8 S={S} vs model")
    ob, deqb = run_bf16(q, k, v)
    assert orc.rel_fro(ob, orc.attention(*deqb)) <= TOL_BF16


@pytest.mark.parametrize("q_gain,kind", [(6.0, "gaussian"), (1.0, "outlier_k"), (12.0, "gaussian")])
def test_fp8_block_scales_engaged(q_gain, kind):
    # peaked scores: many 64-key blocks sit far below the row max, so the
    # per-block power-of-two shift j varies (exercises the scale factors)
    q, k, v = inputs(43, 1, 700, 4, 2, 128, 128, kind=kind, q_gain=q_gain)
    o, codes = run_fp8(q, k, v)
    ref, model = fp8_references(codes)
    e_model, e_ref = orc.rel_fro(o, model), orc.rel_fro(o, ref)
    print(f"fp8 gain={q_gain} {kind}: vs fp64 {e_ref:.3e}  vs model {e_model:.3e}")
    assert e_model <= TOL_FP8_MODEL
    assert e_ref <= TOL_FP8


def test_deferred_reference_max_on_growing_scores():
    """Scores that jump past the kernel's deferral bound (64 binades: a
    rescale), then ~33 binades above the reference (deferred: block shifts
    below 0 and E8M0 scales above 1), fall, then ~78 above it (rescaled), one
    level per KV tile of the FP8 kernel: FP8
    against fp64 attention and the CPU replay with the same deferral rule;
    BF16 on the same values."""
    from test_oracle_pins import _growing_score_case
    qc, kc, vc, qs, ks, vs = _growing_score_case(21, RESCALE_LOG2, fp8_kv_tile(128))
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    o = zyfa.attn_fwd(dev(qc), dev(kc), dev(vc), q_scale=dev(qs), k_scale=dev(ks), v_scale=dev(vs))
    torch.cuda.synchronize()
    o = o.float().cpu().numpy().astype(np.float64)
    ref, model = fp8_references(((qc, qs), (kc, ks), (vc, vs)))
    e_ref, e_model = orc.rel_fro(o, ref), orc.rel_fro(o, model)
    print(f"growing scores fp8: vs fp64 {e_ref:.3e}  vs model {e_model:.3e}")
    assert e_ref <= TOL_FP8 and e_model <= TOL_FP8_MODEL
    deq = [orc.dequantize(x, sc) for x, sc in ((qc, qs), (kc, ks), (vc, vs))]
    ob = zyfa.attn_fwd(*[dev(x).to(torch.bfloat16) for x in deq])   # e4m3 values are exact in bf16
    torch.cuda.synchronize()
    e_b = orc.rel_fro(ob.float().cpu().numpy().astype(np.float64), ref)
    print(f"growing scores bf16: vs fp64 {e_b:.3e}")
    assert e_b <= TOL_BF16


@pytest.mark.parametrize("kind,q_gain", [("outlier_k", 1.0), ("gaussian", 6.0)])
def test_many_units_per_cta(kind, q_gain):
    """512 work units on the persistent grid (several per CTA): unit hand-over
    of O, the epilogue by either softmax group, Q double buffering and, with
    peaked scores, frequent O rescales; sampled rows, FP8 and BF16, repeat
    runs bit-identical."""
    B, S, Hq, Hkv = 2, 2048, 16, 4
    q, k, v = inputs(46, B, S, Hq, Hkv, 128, 128, kind=kind, q_gain=q_gain)
    rows = np.unique(np.concatenate([np.arange(0, S, 37), np.arange(127, S, 128), np.arange(128, S, 128),
                                     [S - 1]])).astype(np.int32)
    o, codes = run_fp8(q, k, v)
    ref, model = fp8_references(codes, rows=rows)
    e_ref, e_model = orc.rel_fro(o[:, rows], ref), orc.rel_fro(o[:, rows], model)
    print(f"many units fp8 {kind} gain={q_gain}: vs fp64 {e_ref:.3e}  vs model {e_model:.3e}")
    assert e_ref <= TOL_FP8 and e_model <= TOL_FP8_MODEL
    check_local(o[:, rows], ref, TOL_FP8, ROW_TOL_FP8, f"many units fp8 {kind} vs fp64", rows)
    check_local(o[:, rows], model, TOL_FP8_MODEL, ROW_TOL_FP8_MODEL, f"many units fp8 {kind} vs model", rows)
    (qc, qs), (kc, ks), (vc, vs) = codes
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    o2 = zyfa.attn_fwd(dev(qc), dev(kc), dev(vc), q_scale=dev(qs), k_scale=dev(ks), v_scale=dev(vs))
    torch.cuda.synchronize()
    assert np.array_equal(o2.float().cpu().numpy().astype(np.float64), o)
    ob, (qb, kb, vb) = run_bf16(q, k, v)
    refb = orc.attention(qb, kb, vb, rows=rows)
    e_b = orc.rel_fro(ob[:, rows], refb)
    print(f"many units bf16 {kind} gain={q_gain}: vs fp64 {e_b:.3e}")
    assert e_b <= TOL_BF16
    check_local(ob[:, rows], refb, TOL_BF16, ROW_TOL_BF16, f"many units bf16 {kind} vs fp64", rows)
    ob2, _ = run_bf16(q, k, v)
    assert np.array_equal(ob2, ob)


@pytest.mark.parametrize("shape", [(1, 512, 2, 2, 128, 128), (2, 700, 4, 2, 128, 128), (1, 300, 2, 2, 192, 128)],
                         ids=lambda s: "x".join(map(str, s)))
def test_fp8_exact_p_ablation(shape):
    """Exact P (ex2 then e4m3) in the same kernel: within the FP8 bar of fp64
    attention, close to the CPU replay of the same route, and no less accurate
    than Lean P on the same codes."""
    import torch
    B, S, Hq, Hkv, Dqk, Dv = shape
    q, k, v = inputs(47, B, S, Hq, Hkv, Dqk, Dv, kind="outlier_k" if Dqk == 128 else "mla")
    o_lean, codes = run_fp8(q, k, v)
    (qc, qs), (kc, ks), (vc, vs) = codes
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    o = zyfa.attn_fwd(dev(qc), dev(kc), dev(vc), q_scale=dev(qs), k_scale=dev(ks), v_scale=dev(vs), exact_p=True)
    torch.cuda.synchronize()
    o = o.float().cpu().numpy().astype(np.float64)
    ref, _ = fp8_references(codes)
    model = orc.fp8_model(qc, kc, vc, qs, ks, vs, p_mode=2, rescale_log2=RESCALE_LOG2, kv_tile=fp8_kv_tile(Dqk))
    e_ref, e_model, e_lean = orc.rel_fro(o, ref), orc.rel_fro(o, model), orc.rel_fro(o_lean, ref)
    print(f"exact-P {shape}: vs fp64 {e_ref:.3e}  vs exact-P model {e_model:.3e}  (Lean P vs fp64 {e_lean:.3e})")
    assert e_ref <= TOL_FP8 and e_model <= TOL_FP8_MODEL
    assert e_ref <= e_lean * 1.05
    assert zyfa.device_status() == zyfa.OK


@pytest.mark.parametrize("shape", [(1, 300, 2, 2, 128, 128), (2, 700, 4, 2, 128, 128), (1, 260, 4, 4, 192, 128)],
                         ids=lambda s: "x".join(map(str, s)))
def test_lse_output(shape):
    """zyfa_attn_fwd_lse: the same O as zyfa_attn_fwd (bit for bit) plus each
    row's log-sum-exp.  BF16 against the fp64 definition on the bf16 inputs;
    FP8 against the CPU replay's own value (same weights) and, within the Lean-P
    weight error, against the fp64 definition on the dequantized inputs."""
    import torch
    B, S, Hq, Hkv, Dqk, Dv = shape
    q, k, v = inputs(49, B, S, Hq, Hkv, Dqk, Dv, kind="outlier_k" if Dqk == 128 else "mla")
    qb, kb, vb = (bf16_round(x).cuda() for x in (q, k, v))
    o_plain = zyfa.attn_fwd(qb, kb, vb)
    o, lse = zyfa.attn_fwd(qb, kb, vb, lse=True)
    torch.cuda.synchronize()
    assert torch.equal(o, o_plain)
    ref = orc.attention_lse(qb.cpu().double().numpy(), kb.cpu().double().numpy())
    e_b = np.abs(lse.cpu().numpy() - ref).max()
    print(f"lse bf16 {shape}: max abs err {e_b:.2e}")
    assert e_b < 2e-3
    o8, codes = run_fp8(q, k, v)
    (qc, qs), (kc, ks), (vc, vs) = codes
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    o8b, lse8 = zyfa.attn_fwd(dev(qc), dev(kc), dev(vc), q_scale=dev(qs), k_scale=dev(ks), v_scale=dev(vs), lse=True)
    torch.cuda.synchronize()
    assert np.array_equal(o8b.float().cpu().numpy().astype(np.float64), o8)
    _, lse_model = orc.fp8_model(qc, kc, vc, qs, ks, vs, rescale_log2=RESCALE_LOG2, return_lse=True,
                                 kv_tile=fp8_kv_tile(Dqk))
    deq = [orc.dequantize(x, sc) for x, sc in codes]
    lse_ref = orc.attention_lse(deq[0], deq[1])
    g = lse8.cpu().numpy()
    d = np.abs(g - lse_model)
    print(f"lse fp8 {shape}: vs replay max {d.max():.2e} median {np.median(d):.1e} mean {d.mean():.1e}  "
          f"vs fp64 {np.abs(g - lse_ref).max():.2e}")
    # A score whose fp32 tensor-core sum and fp64 replay sum straddle an integer
    # of u gets a code one step apart: that weight differs by 2^(1/8), so a row's
    # row sum by at most that factor, its lse by ln 2^(1/8) = 0.0866; such rows
    # are rare (the bulk of rows equals the replay's value).  Against fp64 add
    # Lean P's own per-weight band (2^-1/8, 1.0615]: at most 2 x 0.0866.
    assert d.max() <= 0.087 and np.median(d) <= 1e-5 and d.mean() <= 5e-3
    assert np.abs(g - lse_ref).max() <= 0.18


def test_fp8_hadamard_prepass_path_mla():
    """MLA shape with Q and K rotated block-diagonally (H128 + H64): the same
    bars as without the rotation, which cancels in Q K^T."""
    q, k, v = inputs(48, 1, 400, 4, 4, 192, 128, kind="mla")
    o, codes = run_fp8(q, k, v, hadamard=True)
    ref, model = fp8_references(codes)
    assert orc.rel_fro(o, ref) <= TOL_FP8
    assert orc.rel_fro(o, model) <= TOL_FP8_MODEL
    assert orc.rel_fro(o, orc.attention(q, k, v)) < 0.1


def test_fp8_hadamard_prepass_path():
    q, k, v = inputs(44, 1, 513, 4, 4, 128, 128)
    o, codes = run_fp8(q, k, v, hadamard=True)
    ref, model = fp8_references(codes)
    assert orc.rel_fro(o, ref) <= TOL_FP8
    assert orc.rel_fro(o, model) <= TOL_FP8_MODEL
    # rotation cancels in Q K^T: compare with unquantized fp64 attention too (reported bar)
    unq = orc.attention(q, k, v)
    assert orc.rel_fro(o, unq) < 0.1


def test_zero_q_gives_prefix_means_fp8_and_bf16():
    q, k, v = inputs(45, 1, 260, 2, 2, 128, 128)
    q[:] = 0.0
    o8, codes = run_fp8(q, k, v)
    vd = orc.dequantize(*codes[2])
    pref = np.cumsum(vd, axis=1) / np.arange(1, 261)[None, :, None, None]
    assert orc.rel_fro(o8, pref) <= 2e-3            # equal weights: only bf16 output rounding
    ob, (_, _, vb) = run_bf16(q, k, v)
    prefb = np.cumsum(vb, axis=1) / np.arange(1, 261)[None, :, None, None]
    assert orc.rel_fro(ob, prefb) <= 2e-3


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_deterministic_repeated_runs_and_streams(dtype):
    q, k, v = inputs(46, 1, 1100, 8, 2, 128, 128)
    if dtype == "bf16":
        args = [torch.from_numpy(x).to(torch.bfloat16).cuda() for x in (q, k, v)]
        kw = {}
    else:
        from bf16_causal_prefill_fp8_b200 import zyfa as z
        qc, qs = z.quantize(torch.from_numpy(q).cuda())
        kc, ks = z.quantize(torch.from_numpy(k).cuda())
        vc, vs = z.quantize(torch.from_numpy(v).cuda())
        args, kw = [qc, kc, vc], dict(q_scale=qs, k_scale=ks, v_scale=vs)
    first = zyfa.attn_fwd(*args, **kw).clone()
    s2 = torch.cuda.Stream()
    for i in range(20):
        if i % 2:
            with torch.cuda.stream(s2):
                o = zyfa.attn_fwd(*args, **kw)
            s2.synchronize()
        else:
            o = zyfa.attn_fwd(*args, **kw)
        assert torch.equal(o, first)
    assert zyfa.device_status() == zyfa.OK
