"""Run one workload's kernels a few times, for a profiler to capture.

    python -m bf16_causal_prefill_fp8_b200.profile_case --workload gqa32x8_s16k_outlier --iters 3

Each iteration launches, in order: zyfa_quantize_qkv (zero, amax, codes and
finalize kernels over Q, K and V together), the FP8 attention kernel, then the
BF16 attention kernel on the same bf16 inputs (for a packed-batch workload,
the varlen forms of the same three calls).  --exact-p swaps the FP8 attention
for the exact-P ablation (fixed-length workloads).  Prints nothing but a completion line; timing
numbers come from bench.py, never from a profiled run.
"""
import argparse

import torch

from . import synth, zyfa


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="gqa32x8_s16k_outlier",
                    choices=sorted(synth.WORKLOADS) + sorted(synth.VARLEN_WORKLOADS))
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--hadamard", action="store_true")
    ap.add_argument("--only", choices=["all", "fp8", "bf16"], default="all")
    ap.add_argument("--exact-p", action="store_true",
                    help="the FP8 attention launch is the exact-P ablation (e4m3(ex2(.)) instead of Lean P)")
    args = ap.parse_args()
    if args.workload in synth.VARLEN_WORKLOADS:
        # packed batch: the varlen prepass and varlen attention launches
        wl = synth.VARLEN_WORKLOADS[args.workload]
        lens = synth.varlen_lengths(0, wl["nseq"], wl["lo"], wl["hi"])
        cu = [0]
        for n in lens:
            cu.append(cu[-1] + n)
        q, k, v = synth.make_qkv(0, 1, cu[-1], wl["Hq"], wl["Hkv"], wl["Dqk"], wl["Dv"], wl["kind"])
        dq, dk, dv = (torch.from_numpy(x[0]).to(torch.bfloat16).cuda() for x in (q, k, v))
        quant = lambda: zyfa.quantize_qkv_varlen(dq, dk, dv, cu, hadamard_qk=args.hadamard)
        attn = lambda *t, **kw: zyfa.attn_fwd_varlen(*t, cu, **kw)
    else:
        wl = synth.WORKLOADS[args.workload]
        q, k, v = synth.make_qkv(0, wl["B"], wl["S"], wl["Hq"], wl["Hkv"], wl["Dqk"], wl["Dv"], wl["kind"])
        dq, dk, dv = (torch.from_numpy(x).to(torch.bfloat16).cuda() for x in (q, k, v))
        quant = lambda: zyfa.quantize_qkv(dq, dk, dv, hadamard_qk=args.hadamard)
        attn = zyfa.attn_fwd
    for _ in range(args.iters):
        if args.only in ("all", "fp8"):
            (cq, sq), (ck, sk), (cv, sv) = quant()
            if args.exact_p:
                attn(cq, ck, cv, q_scale=sq, k_scale=sk, v_scale=sv, exact_p=True)
            else:
                attn(cq, ck, cv, q_scale=sq, k_scale=sk, v_scale=sv)
        if args.only in ("all", "bf16"):
            attn(dq, dk, dv)
    torch.cuda.synchronize()
    st = zyfa.device_status()
    print(f"profile_case {args.workload}: {args.iters} iterations done, device status {st}")
    return 0 if st == zyfa.OK else 1


if __name__ == "__main__":
    raise SystemExit(main())
