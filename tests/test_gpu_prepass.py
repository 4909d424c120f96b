"""Prepass (zyfa_quantize) against the oracle's quantizer: codes and scales
must match byte for byte, with and without the Hadamard rotation."""
import numpy as np
import pytest
import torch

from bf16_causal_prefill_fp8_b200 import synth, zyfa
from oracle import oracle as orc

from helpers import bf16_round, quantize_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape,hadamard", [((1, 200, 3, 128), False), ((1, 200, 3, 128), True),
                                            ((2, 77, 4, 192), False), ((3, 1, 5, 128), True),
                                            ((1, 1000, 8, 128), True), ((2, 129, 2, 64), False),
                                            ((2, 77, 4, 192), True), ((1, 300, 3, 192), True)])
@pytest.mark.parametrize("as_bf16", [False, True])
def test_quantize_bit_exact(shape, hadamard, as_bf16):
    x = synth.gaussian(21, 1, shape) * np.float32(3.0)
    x[0, :, 0, :] *= np.float32(50.0)                     # heads with different ranges
    if shape[2] > 2:
        x[-1, :, 2, :] = 0.0                              # an all-zero head: scale 1
    codes, scale = quantize_gpu(x, hadamard=hadamard, as_bf16=as_bf16)
    xin = bf16_round(x).float().numpy() if as_bf16 else x
    rc, rs = orc.quantize(xin, hadamard=hadamard)
    assert np.array_equal(scale.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    got = codes.cpu().numpy()
    assert np.array_equal(got, rc), f"{np.count_nonzero(got != rc)} codes differ"


def test_quantize_outlier_channels_and_subnormals():
    x = synth.gaussian(22, 2, (1, 333, 4, 128))
    std, _ = synth.outlier_channel_std(22, 4, 128)
    x = (x * std[None, None]).astype(np.float32)
    for had in (False, True):
        codes, scale = quantize_gpu(x, hadamard=had)
        rc, rs = orc.quantize(x, hadamard=had)
        assert np.array_equal(scale.cpu().numpy().view(np.uint32), rs.view(np.uint32))
        assert np.array_equal(codes.cpu().numpy(), rc)


@pytest.mark.parametrize("B,S,Hq,Hkv,Dqk,Dv,hadamard", [(1, 300, 8, 2, 128, 128, False),
                                                        (2, 129, 4, 4, 128, 128, True),
                                                        (1, 77, 6, 2, 192, 128, False),
                                                        (1, 77, 6, 2, 192, 128, True),
                                                        (1, 2048, 32, 8, 128, 128, True),
                                                        (3, 5, 2, 1, 128, 128, False)])
@pytest.mark.parametrize("as_bf16", [False, True])
def test_quantize_qkv_equals_three_calls_and_oracle(B, S, Hq, Hkv, Dqk, Dv, hadamard, as_bf16):
    """zyfa_quantize_qkv (one grid for Q, K and V per step) gives the oracle's
    codes and scales, byte for byte, like three zyfa_quantize calls."""
    import torch
    from bf16_causal_prefill_fp8_b200 import zyfa
    q, k, v = synth.make_qkv(31, B, S, Hq, Hkv, Dqk, Dv, "outlier_k")
    q[0, :, 0, :] *= np.float32(40.0)
    to = (lambda x: bf16_round(x).cuda()) if as_bf16 else (lambda x: torch.from_numpy(x).cuda())
    got = zyfa.quantize_qkv(to(q), to(k), to(v), hadamard_qk=hadamard)
    torch.cuda.synchronize()
    for (c, sc), x, had in zip(got, (q, k, v), (hadamard, hadamard, False)):
        xin = bf16_round(x).float().numpy() if as_bf16 else x
        rc, rs = orc.quantize(xin, hadamard=had)
        assert np.array_equal(sc.cpu().numpy().view(np.uint32), rs.view(np.uint32))
        assert np.array_equal(c.cpu().numpy(), rc)


def test_quantize_quotients_at_e4m3_midpoints():
    """Inputs whose quotient by the head scale lands exactly on, or one fp32 ulp
    either side of, every rounding midpoint between adjacent e4m3 values: a
    quotient off by one ulp flips the code here.  The scale is uneven
    (amax = 448 * 1.3717), so the division is not exact."""
    vals = np.sort(np.unique(np.abs(orc.e4m3_values()[np.isfinite(orc.e4m3_values())]))).astype(np.float64)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)          # exact in fp32
    amax = np.float32(448.0 * 1.3717)
    s = np.float32(amax / np.float32(448.0))
    xs = []
    for m in mids:
        x = np.float32(m * s)
        xs += [np.nextafter(x, np.float32(-np.inf)), x, np.nextafter(x, np.float32(np.inf))]
    xs = np.array(xs, dtype=np.float32)
    xs = np.concatenate([xs, -xs, [amax]])
    n = (len(xs) + 127) // 128 * 128
    row = np.zeros(n, dtype=np.float32); row[:len(xs)] = xs
    x = row.reshape(1, n // 128, 1, 128)
    codes, scale = quantize_gpu(x)
    rc, rs = orc.quantize(x)
    assert np.array_equal(scale.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    got = codes.cpu().numpy()
    assert np.array_equal(got, rc), f"{np.count_nonzero(got != rc)} codes differ"


@pytest.mark.parametrize("tiny", [1e-37, 3e-39])
def test_quantize_tiny_head_uses_plain_division(tiny):
    """A head whose scale amax/448 has no normal reciprocal (below 2^-120, down
    into fp32 subnormals) makes its CTAs take the IEEE-division path for every
    head they hold; codes and scales stay byte-exact, for that head and its
    normal neighbours, in the one-tensor and the fused Q/K/V prepass."""
    x = synth.gaussian(23, 2, (2, 260, 3, 128)).astype(np.float32)
    x[:, :, 1] *= np.float32(tiny)
    codes, scale = quantize_gpu(x)
    rc, rs = orc.quantize(x)
    assert np.array_equal(scale.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert float(rs.reshape(2, 3)[0, 1]) < 2.0 ** -120
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    got = zyfa.quantize_qkv(t(x), t(x[:, :, :1]), t(x[:, :, 1:2]))
    torch.cuda.synchronize()
    for (c, sc), xi in zip(got, (x, x[:, :, :1], x[:, :, 1:2])):
        rci, rsi = orc.quantize(np.ascontiguousarray(xi))
        assert np.array_equal(sc.cpu().numpy().view(np.uint32), rsi.view(np.uint32))
        assert np.array_equal(c.cpu().numpy(), rci)
