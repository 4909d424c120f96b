"""The pages' workloads at full size, in the launch configuration bench.py
times (fused Q/K/V prepass, then the FP8 attention; the BF16 attention on the
same bf16 inputs), checked on sampled query rows the oracle computes one by
one: a seeded row inside every 128-row query tile plus tile-edge rows, for
every head.  Beside the whole-tensor bound, every head and every sampled
(row, head) output vector has its own bound, so one corrupted tile of one head
fails.  The FP8 output is also compared per row with the oracle's replay of
the FP8 pipeline on the same codes.  The prepass codes and scales are compared
in full."""
import numpy as np
import pytest
import torch

from bf16_causal_prefill_fp8_b200 import synth, zyfa
from oracle import oracle as orc

from helpers import (RESCALE_LOG2, ROW_TOL_BF16, ROW_TOL_FP8, ROW_TOL_FP8_MODEL, TOL_BF16, TOL_FP8,
                     TOL_FP8_MODEL, check_local, fp8_kv_tile, tile_rows)

pytestmark = pytest.mark.gpu

WORKLOADS = [  # name, B, S, Hq, Hkv, Dqk, Dv, kind, hadamard
    ("gqa32x8_s16k_outlier", 1, 16384, 32, 8, 128, 128, "outlier_k", False),
    ("mha32_s32k", 1, 32768, 32, 32, 128, 128, "gaussian", False),
    ("mla16_s16k_192_128", 1, 16384, 16, 16, 192, 128, "mla", False),
    ("sweep_s64k_hadamard", 1, 65536, 32, 32, 128, 128, "gaussian", True),
]


@pytest.mark.parametrize("wl", WORKLOADS, ids=lambda w: w[0])
def test_full_size_sampled_parity(wl):
    name, B, S, Hq, Hkv, Dqk, Dv, kind, hadamard = wl
    tb = [torch.from_numpy(x).to(torch.bfloat16) for x in synth.make_qkv(0, B, S, Hq, Hkv, Dqk, Dv, kind)]
    dq, dk, dv = (t.cuda() for t in tb)
    (cq, sq), (ck, sk), (cv, sv) = zyfa.quantize_qkv(dq, dk, dv, hadamard_qk=hadamard)
    o8 = zyfa.attn_fwd(cq, ck, cv, q_scale=sq, k_scale=sk, v_scale=sv)
    ob = zyfa.attn_fwd(dq, dk, dv)
    torch.cuda.synchronize()
    assert zyfa.device_status() == zyfa.OK
    del dq, dk, dv
    xs = [t.float().numpy() for t in tb]
    codes = [orc.quantize(xs[0], hadamard), orc.quantize(xs[1], hadamard), orc.quantize(xs[2], False)]
    for (gc, gs), (rc, rs) in zip(((cq, sq), (ck, sk), (cv, sv)), codes):
        assert np.array_equal(gs.cpu().numpy().view(np.uint32), rs.view(np.uint32))
        assert np.array_equal(gc.cpu().numpy(), rc)
    rows = tile_rows(S, 3)
    deq = [orc.dequantize(c, s) for c, s in codes]
    ref8 = orc.attention(*deq, rows=rows)
    del deq
    (qc, qs), (kc, ks), (vc, vs) = codes
    model = orc.fp8_model(qc, kc, vc, qs, ks, vs, rows=rows, rescale_log2=RESCALE_LOG2,
                          kv_tile=fp8_kv_tile(qc.shape[3]))
    got8 = o8.float().cpu().numpy()[:, rows].astype(np.float64)
    err8, err8m = orc.rel_fro(got8, ref8), orc.rel_fro(got8, model)
    refb = orc.attention(*[x.astype(np.float64) for x in xs], rows=rows)
    gotb = ob.float().cpu().numpy()[:, rows].astype(np.float64)
    errb = orc.rel_fro(gotb, refb)
    print(f"{name}: {len(rows)} rows x {Hq} heads; fp8 vs fp64 (dequantized) {err8:.3e}, "
          f"vs replay {err8m:.3e}; bf16 {errb:.3e}")
    assert err8 <= TOL_FP8, err8
    assert err8m <= TOL_FP8_MODEL, err8m
    assert errb <= TOL_BF16, errb
    check_local(got8, ref8, TOL_FP8, ROW_TOL_FP8, f"{name} fp8 vs fp64", rows)
    check_local(got8, model, TOL_FP8_MODEL, ROW_TOL_FP8_MODEL, f"{name} fp8 vs replay", rows)
    check_local(gotb, refb, TOL_BF16, ROW_TOL_BF16, f"{name} bf16 vs fp64", rows)
