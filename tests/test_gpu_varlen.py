"""Packed (variable-length) batches through zyfa_attn_fwd_varlen and the
varlen prepass, against the oracle's per-sequence references, and bit for bit
against the fixed-length kernel run on each sequence alone (each unit's
arithmetic depends only on its own sequence, whatever CTA runs it).

Lengths cover empty sequences, one row, exact tiles, a tile plus one and
ragged tails, in shuffled order so the longest-first schedule reorders them."""
import random

import numpy as np
import pytest
import torch

from bf16_causal_prefill_fp8_b200 import synth, zyfa
from oracle import oracle as orc

from helpers import RESCALE_LOG2, TOL_BF16, TOL_FP8, TOL_FP8_MODEL, bf16_round, fp8_kv_tile

pytestmark = pytest.mark.gpu

LENS_A = [300, 0, 1, 128, 129, 1000, 77]
LENS_B = [random.Random(5).randint(0, 700) for _ in range(20)]


def cu_of(lens):
    return [0] + list(np.cumsum(lens).astype(int))


def packed(seed, lens, Hq, Hkv, Dqk, Dv, kind="gaussian"):
    q, k, v = synth.make_qkv(seed, 1, max(1, int(sum(lens))), Hq, Hkv, Dqk, Dv, kind)
    T = int(sum(lens))
    return q[0, :T], k[0, :T], v[0, :T]


def spans(lens):
    cu = cu_of(lens)
    return [(s, cu[s], cu[s + 1]) for s in range(len(lens)) if cu[s + 1] > cu[s]]


def gpu_bf16(x):
    return bf16_round(x).cuda()


SHAPES = [(4, 2, 128, 128, "gaussian"), (2, 2, 192, 128, "mla"), (8, 1, 128, 128, "outlier_k")]


@pytest.mark.parametrize("lens", [LENS_A, LENS_B], ids=["edge", "random20"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s[:4])))
def test_bf16_varlen_parity_and_equal_to_single_sequence(lens, shape):
    Hq, Hkv, Dqk, Dv, kind = shape
    q, k, v = packed(51, lens, Hq, Hkv, Dqk, Dv, kind)
    dq, dk, dv = gpu_bf16(q), gpu_bf16(k), gpu_bf16(v)
    o = zyfa.attn_fwd_varlen(dq, dk, dv, cu_of(lens))
    torch.cuda.synchronize()
    assert zyfa.device_status() == zyfa.OK
    qd, kd, vd = (t.double().cpu().numpy() for t in (dq, dk, dv))
    ref = orc.attention_varlen(qd, kd, vd, cu_of(lens))
    got = o.float().cpu().numpy().astype(np.float64)
    for s, r0, r1 in spans(lens):
        err = orc.rel_fro(got[r0:r1], ref[r0:r1])
        assert err <= TOL_BF16, (s, err)
        single = zyfa.attn_fwd(dq[None, r0:r1].contiguous(), dk[None, r0:r1].contiguous(),
                               dv[None, r0:r1].contiguous())
        assert torch.equal(single[0], o[r0:r1]), s


@pytest.mark.parametrize("hadamard", [False, True])
@pytest.mark.parametrize("lens", [LENS_A, LENS_B], ids=["edge", "random20"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s[:4])))
def test_fp8_varlen_parity_and_equal_to_single_sequence(lens, shape, hadamard):
    Hq, Hkv, Dqk, Dv, kind = shape
    q, k, v = packed(52, lens, Hq, Hkv, Dqk, Dv, kind)
    cu = cu_of(lens)
    dq, dk, dv = (torch.from_numpy(np.ascontiguousarray(t)).cuda() for t in (q, k, v))
    (qc, qs), (kc, ks), (vc, vs) = zyfa.quantize_qkv_varlen(dq, dk, dv, cu, hadamard_qk=hadamard)
    o, lse = zyfa.attn_fwd_varlen(qc, kc, vc, cu, q_scale=qs, k_scale=ks, v_scale=vs, lse=True)
    torch.cuda.synchronize()
    assert zyfa.device_status() == zyfa.OK
    # the prepass: bit-identical to the oracle's per-sequence quantization
    ref_q = [orc.quantize_varlen(q, cu, hadamard), orc.quantize_varlen(k, cu, hadamard),
             orc.quantize_varlen(v, cu, False)]
    for (gc, gs), (rc, rs) in zip(((qc, qs), (kc, ks), (vc, vs)), ref_q):
        assert np.array_equal(gc.cpu().numpy(), rc)
        assert np.array_equal(gs.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    (rqc, rqs), (rkc, rks), (rvc, rvs) = ref_q
    table = orc.e4m3_values()
    seq = np.repeat(np.arange(len(lens)), lens)
    deq = [table[c] * s_[seq][:, :, None].astype(np.float64) for c, s_ in ((rqc, rqs), (rkc, rks), (rvc, rvs))]
    ref = orc.attention_varlen(*deq, cu)
    model = orc.fp8_model_varlen(rqc, rkc, rvc, rqs, rks, rvs, cu, rescale_log2=RESCALE_LOG2,
                                 kv_tile=fp8_kv_tile(rqc.shape[2]))
    got = o.float().cpu().numpy().astype(np.float64)
    for s, r0, r1 in spans(lens):
        err, err_m = orc.rel_fro(got[r0:r1], ref[r0:r1]), orc.rel_fro(got[r0:r1], model[r0:r1])
        assert err <= TOL_FP8, (s, err)
        assert err_m <= TOL_FP8_MODEL, (s, err_m)
        single, single_lse = zyfa.attn_fwd(qc[None, r0:r1].contiguous(), kc[None, r0:r1].contiguous(),
                                           vc[None, r0:r1].contiguous(), q_scale=qs[s:s + 1].contiguous(),
                                           k_scale=ks[s:s + 1].contiguous(), v_scale=vs[s:s + 1].contiguous(),
                                           lse=True)
        assert torch.equal(single[0], o[r0:r1]), s
        assert torch.equal(single_lse[0], lse[:, r0:r1]), s


@pytest.mark.parametrize("fp8", [False, True])
def test_equal_lengths_equal_the_fixed_length_batch(fp8):
    """Three sequences of 777 rows: the same schedule, unit for unit, as the
    fixed-length launch with B = 3, so the outputs are bit-identical."""
    B, S, Hq, Hkv, D = 3, 777, 4, 2, 128
    q, k, v = synth.make_qkv(53, B, S, Hq, Hkv, D, D)
    if fp8:
        dq, dk, dv = (torch.from_numpy(t).cuda() for t in (q, k, v))
        (qc, qs), (kc, ks), (vc, vs) = zyfa.quantize_qkv(dq, dk, dv)
        fixed = zyfa.attn_fwd(qc, kc, vc, q_scale=qs, k_scale=ks, v_scale=vs)
        var = zyfa.attn_fwd_varlen(qc.view(B * S, Hq, D), kc.view(B * S, Hkv, D), vc.view(B * S, Hkv, D),
                                   [0, S, 2 * S, 3 * S], q_scale=qs, k_scale=ks, v_scale=vs)
    else:
        dq, dk, dv = gpu_bf16(q), gpu_bf16(k), gpu_bf16(v)
        fixed = zyfa.attn_fwd(dq, dk, dv)
        var = zyfa.attn_fwd_varlen(dq.view(B * S, Hq, D), dk.view(B * S, Hkv, D), dv.view(B * S, Hkv, D),
                                   [0, S, 2 * S, 3 * S])
    torch.cuda.synchronize()
    assert torch.equal(fixed.view(B * S, Hq, D), var)


@pytest.mark.parametrize("hadamard,D", [(False, 128), (True, 128), (True, 192), (False, 64)])
def test_quantize_varlen_equals_single_sequence_prepass(hadamard, D):
    H = 3
    x = synth.gaussian(54, 1, (int(sum(LENS_B)), H, D)) * np.float32(2.5)
    dx = gpu_bf16(x)
    codes, scale = zyfa.quantize_varlen(dx, cu_of(LENS_B), hadamard=hadamard)
    torch.cuda.synchronize()
    for s, r0, r1 in spans(LENS_B):
        c1, s1 = zyfa.quantize(dx[None, r0:r1].contiguous(), hadamard=hadamard)
        assert torch.equal(c1[0], codes[r0:r1]), s
        assert torch.equal(s1[0], scale[s]), s
    empty = [s for s, n in enumerate(LENS_B) if n == 0]
    for s in empty:
        assert torch.all(scale[s] == 1.0)
    rc, rs = orc.quantize_varlen(dx.float().cpu().numpy(), cu_of(LENS_B), hadamard)
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scale.cpu().numpy().view(np.uint32), rs.view(np.uint32))


def test_384_sequences_and_a_long_one():
    """The largest table (384 sequences, one of them 9000 rows): sampled
    sequences bit-identical to single-sequence launches, the long one checked
    against the oracle on sampled rows."""
    rng = random.Random(7)
    lens = [rng.randint(0, 200) for _ in range(383)] + [9000]
    rng.shuffle(lens)
    Hq, Hkv, D = 4, 2, 128
    q, k, v = packed(55, lens, Hq, Hkv, D, D)
    dq, dk, dv = gpu_bf16(q), gpu_bf16(k), gpu_bf16(v)
    cu = cu_of(lens)
    o = zyfa.attn_fwd_varlen(dq, dk, dv, cu)
    torch.cuda.synchronize()
    assert zyfa.device_status() == zyfa.OK
    sp = spans(lens)
    for s, r0, r1 in rng.sample(sp, 12) + [t for t in sp if t[2] - t[1] == 9000]:
        single = zyfa.attn_fwd(dq[None, r0:r1].contiguous(), dk[None, r0:r1].contiguous(),
                               dv[None, r0:r1].contiguous())
        assert torch.equal(single[0], o[r0:r1]), s
    s, r0, r1 = next(t for t in sp if t[2] - t[1] == 9000)
    rows = [0, 1, 127, 128, 4500, 8999]
    qd, kd, vd = (t[r0:r1].double().cpu().numpy()[None] for t in (dq, dk, dv))
    ref = orc.attention(qd, kd, vd, rows=rows)[0]
    got = o[r0:r1].float().cpu().numpy().astype(np.float64)[rows]
    assert orc.rel_fro(got, ref) <= TOL_BF16


def test_all_empty_batch():
    """cu_seqlens all zero: nothing is launched for the attention; the prepass
    writes scale 1.0 for every (empty) sequence."""
    e = torch.empty((0, 2, 128), dtype=torch.bfloat16, device="cuda")
    o = zyfa.attn_fwd_varlen(e, e, e, [0, 0, 0])
    codes, scale = zyfa.quantize_varlen(e, [0, 0, 0])
    torch.cuda.synchronize()
    assert o.shape == (0, 2, 128) and codes.shape == (0, 2, 128)
    assert torch.equal(scale, torch.ones((2, 2), device="cuda"))


def test_binding_rejects_row_count_mismatch():
    x = torch.zeros((10, 2, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        zyfa.attn_fwd_varlen(x, x, x, [0, 4, 11])
    with pytest.raises(ValueError):
        zyfa.quantize_varlen(x, [0, 9])
