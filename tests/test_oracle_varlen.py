"""Pins of the oracle's packed-batch (variable-length) functions against
computations that do not go through them: one masked attention over the whole
packed batch (torch, fp64) with a block-diagonal causal mask, torch's
logsumexp over the same masked scores, per-sequence amax scales in numpy, and
the exact-weight model equal to the fp64 definition on dequantized inputs."""
import numpy as np
import pytest
import torch

from bf16_causal_prefill_fp8_b200 import synth
from oracle import oracle as orc

LENS = [5, 0, 1, 130, 64, 129]


def cu_of(lens):
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)


def packed(seed, lens, Hq, Hkv, Dqk, Dv):
    q, k, v = synth.make_qkv(seed, 1, int(sum(lens)), Hq, Hkv, Dqk, Dv)
    return q[0], k[0], v[0]


def block_causal_mask(lens):
    """mask[i, j]: key j visible to query i (same sequence, j <= i)."""
    seq = np.repeat(np.arange(len(lens)), lens)
    idx = np.arange(len(seq))
    return (seq[:, None] == seq[None, :]) & (idx[None, :] <= idx[:, None])


def torch_masked(q, k, v, mask):
    Hq, Hkv = q.shape[1], k.shape[1]
    g = Hq // Hkv
    qt = torch.from_numpy(q.astype(np.float64)).permute(1, 0, 2)
    kt = torch.from_numpy(k.astype(np.float64)).permute(1, 0, 2).repeat_interleave(g, 0)
    vt = torch.from_numpy(v.astype(np.float64)).permute(1, 0, 2).repeat_interleave(g, 0)
    m = torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m)
    s = (qt @ kt.transpose(1, 2)) / np.sqrt(q.shape[2])
    lse = torch.logsumexp(s.masked_fill(~m, float("-inf")), dim=-1)
    return o.permute(1, 0, 2).numpy(), lse.numpy()


@pytest.mark.parametrize("Hq,Hkv,Dqk,Dv", [(4, 2, 16, 8), (2, 2, 192, 128)])
def test_attention_varlen_equals_one_block_diagonal_masked_attention(Hq, Hkv, Dqk, Dv):
    q, k, v = packed(21, LENS, Hq, Hkv, Dqk, Dv)
    cu = cu_of(LENS)
    o = orc.attention_varlen(q, k, v, cu)
    ref, ref_lse = torch_masked(q, k, v, block_causal_mask(LENS))
    assert np.allclose(o, ref, atol=1e-12, rtol=1e-10)
    lse = orc.attention_lse_varlen(q, k, cu)
    assert np.allclose(lse, ref_lse, atol=1e-12, rtol=1e-12)
    # the first row of every non-empty sequence is its own V row
    g = Hq // Hkv
    for r0, n in zip(cu[:-1], LENS):
        if n:
            assert np.allclose(o[r0], np.repeat(v[r0], g, axis=0), atol=1e-15)


def test_quantize_varlen_scales_are_per_sequence_amax():
    H, D = 3, 128
    x = synth.gaussian(5, 1, (int(sum(LENS)), H, D)) * np.float32(3.0)
    cu = cu_of(LENS)
    codes, scale = orc.quantize_varlen(x, cu)
    assert scale.shape == (len(LENS), H)
    for s, (r0, r1) in enumerate(zip(cu[:-1], cu[1:])):
        if r1 == r0:
            assert np.all(scale[s] == np.float32(1.0))      # amax 0: the scale rule's special case
            continue
        amax = np.abs(x[r0:r1]).max(axis=(0, 2)).astype(np.float32)
        assert np.array_equal(scale[s], (amax / np.float32(448.0)).astype(np.float32))
        # codes decode to within e4m3's half-ulp of x / scale (relative 2^-4, or the subnormal step)
        val = orc.e4m3_values()[codes[r0:r1]]
        want = x[r0:r1] / scale[s][None, :, None].astype(np.float64)
        assert np.all(np.abs(val - want) <= np.maximum(np.abs(want) * 2.0 ** -4, 2.0 ** -10) + 1e-12)


def test_fp8_model_varlen_exact_weights_equal_definition():
    lens = [140, 3, 0, 70]
    Hq, Hkv, D = 2, 1, 128
    q, k, v = packed(8, lens, Hq, Hkv, D, D)
    cu = cu_of(lens)
    (qc, qs), (kc, ks), (vc, vs) = (orc.quantize_varlen(t, cu) for t in (q, k, v))
    table = orc.e4m3_values()
    seq = np.repeat(np.arange(len(lens)), lens)

    def deq(c, s):
        return table[c] * s[seq][:, :, None].astype(np.float64)

    o, lse = orc.fp8_model_varlen(qc, kc, vc, qs, ks, vs, cu, p_mode=1, return_lse=True)
    ref, ref_lse = torch_masked(deq(qc, qs), deq(kc, ks), deq(vc, vs), block_causal_mask(lens))
    assert orc.rel_fro(o, ref) < 1e-6
    assert np.max(np.abs(lse - ref_lse)) < 1e-6
