"""Benchmark: causal prefill attention TFLOP/s on one B200 (or N, weak scaling).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Default workload: the pages' GQA configuration at S = 16K (B=1, Hq=32, Hkv=8,
D=128, K with heavy-tailed outlier channels), seeded synthetic inputs resident
in HBM as bf16.  One step of the headline (FP8) path = the whole hot path:
quantize Q, K, V (bf16 -> e4m3 + per-head scales) and the FP8 Lean-P causal
attention forward.  The BF16 path (one bf16 attention forward on the same
inputs) is timed the same way and reported under "bf16".  L2 is flushed
(256 MiB write, outside the timed events) before every timed step.

Also in the default line (each can be switched off):
  - tensor-core GEMM peaks measured in the same run (cuBLAS bf16 and e4m3
    8192^3, burst and sustained): the denominators of the roofline fractions;
  - a sustained leg: each attention kernel back to back for a few seconds with
    the SM clock and power sampled every 20 ms (TFLOP/s at sustained clock,
    TFLOP per joule);
  - the exact-P ablation of the FP8 kernel, timed and checked like Lean P;
  - the pages' other shapes (MHA 32K, the MLA 192/128 shape, a packed batch of
    32 variable-length sequences), each with its own roofline and sampled parity.

FLOPs: 2 * B * Hq * (S^2 / 2) * (Dqk + Dv) per attention (FlashAttention's
causal convention).  Under torchrun one global problem of world x B batch
entries is split into contiguous runs of (batch, kv head) slots, one run per
rank (weak scaling, no collective on the data path); rank 0 prints one JSON
line.  With --impl reference the CPU oracle (plain C, fp64) is timed instead,
on a bounded sample of rows.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bf16_causal_prefill_fp8_b200 import shard, synth  # noqa: E402

METRIC = "causal prefill attn TFLOP/s (FP8 e4m3 & BF16, D=128, S=16K) and % of B200 peak"
DEFAULT_WORKLOAD = "gqa32x8_s16k_outlier"
EXTRA_WORKLOADS = "mha32_s32k,mla16_s16k_192_128,varlen_gqa32x8_mix32"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DATASHEET = {"bf16": 2250.0, "fp8": 4500.0}
FP8_PER_BF16 = 2.0        # nominal dense FP8 / BF16 tensor throughput ratio on B200
FLOP_PER_CLK_SM = {"bf16": 8192, "fp8": 16384}   # dense tensor-core rate per SM per clock
SMS = 148


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampled every 100 ms while the timed region runs."""
    FIELDS = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id):
        self.bus_id = (bus_id or "").lower()
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            if self.bus_id and self.bus_id[-12:] not in f[1].lower():
                continue
            rows.append(f)
        if not rows:
            return None
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        pw = [float(r[4]) for r in rows if r[4].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[6:10]) if v.lower().startswith("active")})
        load = [s for s in sm if s > 0.3 * (max(mx) if mx else 1)] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "power_w_median": statistics.median(pw) if pw else None, "reasons": reasons,
                "samples": len(rows)}


class NvmlSampler:
    """SM clock, its maximum, board power and the active clock-event reasons of
    one GPU, sampled every 20 ms by NVML on a background thread while the
    timed region runs.  stop() summarises like ClockSampler.stop()."""
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, bus_id, period=0.02):
        import pynvml
        self.nv = pynvml
        pynvml.nvmlInit()
        self.h = None
        want = (bus_id or "").lower()
        for i in range(pynvml.nvmlDeviceGetCount()):
            h = pynvml.nvmlDeviceGetHandleByIndex(i)
            bid = pynvml.nvmlDeviceGetPciInfo(h).busId
            bid = bid.decode() if isinstance(bid, bytes) else bid
            if want and bid.lower()[-12:] == want[-12:]:
                self.h = h
        if self.h is None:
            raise RuntimeError(f"no NVML device with bus id {bus_id}")
        self.period = period
        self.rows = []
        self.stop_ev = threading.Event()
        self.th = None

    def _loop(self):
        nv, h = self.nv, self.h
        while not self.stop_ev.is_set():
            try:
                self.rows.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                  nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM),
                                  nv.nvmlDeviceGetPowerUsage(h) / 1000.0,
                                  nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
            except Exception:   # a failed sample is skipped, not fatal
                pass
            time.sleep(self.period)

    def start(self):
        self.th = threading.Thread(target=self._loop, daemon=True)
        self.th.start()

    def stop(self):
        self.stop_ev.set()
        if self.th:
            self.th.join(timeout=5)
        if not self.rows:
            return None
        mx = max(r[1] for r in self.rows)
        load = [r for r in self.rows if r[0] > 0.3 * mx] or self.rows
        reasons = sorted({n for r in load for n, bit in self.REASONS if r[3] & bit})
        return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": mx,
                "power_w_median": statistics.median(r[2] for r in load), "reasons": reasons,
                "samples": len(self.rows), "source": "nvml, 20 ms"}


def make_sampler(bus):
    """NVML sampling where the library answers, else nvidia-smi (100 ms)."""
    try:
        return NvmlSampler(bus)
    except Exception:
        return ClockSampler(bus)


# ----------------------------------------------------------------- CPU oracle legs

def sample_rows(S, n):
    base = {0, 1, S - 1, S // 2}
    for t in range(1, (S + 127) // 128):
        if len(base) >= n // 2:
            break
        base.update({128 * t - 1, 128 * t})
    rng = np.random.default_rng(7)
    extra = rng.choice(S, size=max(0, min(S, n) - len(base)), replace=False)
    rows = sorted({int(r) for r in base if 0 <= r < S} | {int(r) for r in extra})
    return np.array(rows[:n] if len(rows) > n else rows, dtype=np.int32)


def row_flops(rows, Hq, Dqk, Dv, B):
    return float(B * Hq * sum(2.0 * (int(i) + 1) * (Dqk + Dv) for i in rows))


def e2e_pipelined(torch, pin, bufs, run_step, outs, host_outs, steps):
    """End-to-end steps with copies overlapped: step i's H2D (copy stream)
    runs beside step i-1's compute (current stream) and step i-2's D2H (D2H
    stream); every step still copies its inputs in and its output out.  Buffer
    set i % 2 is rewritten only after step i-2's compute has read it, and
    output i % 2 only after step i-2's D2H has read it.  Returns ms per step:
    events on the current stream around the loop, which waits for the other
    streams' last copies."""
    main = torch.cuda.current_stream()
    cp, dh = torch.cuda.Stream(), torch.cuda.Stream()
    h2d = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    d2h = [torch.cuda.Event() for _ in range(2)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(main)
    cp.wait_event(e0)
    dh.wait_event(e0)
    for i in range(steps):
        s = i % 2
        if i >= 2:
            cp.wait_event(done[s])
        with torch.cuda.stream(cp):
            for dst, src in zip(bufs[s], pin):
                dst.copy_(src, non_blocking=True)
        h2d[s].record(cp)
        main.wait_event(h2d[s])
        if i >= 2:
            main.wait_event(d2h[s])
        run_step(s)
        done[s].record(main)
        dh.wait_event(done[s])
        with torch.cuda.stream(dh):
            host_outs[s].copy_(outs[s], non_blocking=True)
        d2h[s].record(dh)
    for s in range(min(steps, 2)):
        main.wait_event(d2h[s])
    e1.record(main)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def max_head_rel_fro(got, ref):
    """Largest per-head relative Frobenius error; arrays [..., H, D] with the
    head axis second to last."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    H = ref.shape[-2]
    errs = []
    for h in range(H):
        g, r = got[..., h, :], ref[..., h, :]
        errs.append(float(np.linalg.norm((g - r).ravel()) / np.linalg.norm(r.ravel())))
    return max(errs)


def oracle_inputs(wl, seed, xq, xk, xv, hadamard=False):
    """The oracle's own quantization of the bf16 inputs (widened to fp32)."""
    from oracle import oracle as orc
    out = []
    for x, had in ((xq, hadamard), (xk, hadamard), (xv, False)):
        c, s = orc.quantize(x, hadamard=had)
        out.append((c, s))
    return out


def time_oracle_rows(wl, codes, rows):
    from oracle import oracle as orc
    (qc, qs), (kc, ks), (vc, vs) = codes
    deq = (orc.dequantize(qc, qs), orc.dequantize(kc, ks), orc.dequantize(vc, vs))
    t0 = time.perf_counter()
    o = orc.attention(*deq, rows=rows)
    dt = time.perf_counter() - t0
    return o, dt, orc.num_threads(), deq


CPU_BASELINE_SECONDS = 12.0   # CPU work the oracle baseline is timed on (a bounded sample)


def time_oracle_baseline(deq, S, first_rows, first_dt, Hq, Dqk, Dv, B):
    """The oracle on the host cores over a bounded row sample of the workload:
    the parity rows plus further seeded rows, sized from the measured rate to
    about CPU_BASELINE_SECONDS of work.  Returns (TFLOP/s, rows, seconds)."""
    from oracle import oracle as orc
    fl0 = row_flops(first_rows, Hq, Dqk, Dv, B)
    rate = fl0 / max(first_dt, 1e-6)
    want = CPU_BASELINE_SECONDS * rate - fl0
    if want <= 0:
        return fl0 / first_dt / 1e12, len(first_rows), first_dt
    rng = np.random.default_rng(11)
    mean_row = 2.0 * (S / 2) * (Dqk + Dv) * B * Hq
    n = int(min(S, max(1, want / mean_row)))
    extra = np.sort(rng.choice(S, size=n, replace=False)).astype(np.int32)
    t0 = time.perf_counter()
    orc.attention(*deq, rows=extra)
    dt = time.perf_counter() - t0
    fl = fl0 + row_flops(extra, Hq, Dqk, Dv, B)
    return fl / (first_dt + dt) / 1e12, len(first_rows) + n, first_dt + dt


# ----------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(synth.WORKLOADS) + sorted(synth.VARLEN_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--sustained", "--energy", type=float, default=2.0, metavar="SECONDS", dest="sustained",
                    help="run each attention kernel back to back for SECONDS under 20 ms clock / power sampling "
                         "and report sustained TFLOP/s, SM clock and TFLOP per joule (0 = skip)")
    ap.add_argument("--peaks", type=float, default=2.0, metavar="SECONDS",
                    help="measure the cuBLAS bf16 and e4m3 GEMM peaks (8192^3) in this run: burst, and back to "
                         "back for SECONDS (0 = skip: the driver-measured or fallback figures stand)")
    ap.add_argument("--no-exact-p", action="store_true",
                    help="skip the exact-P ablation (ex2 then e4m3 P) of the FP8 attention")
    ap.add_argument("--also", default=EXTRA_WORKLOADS,
                    help="comma-separated further workloads reported under 'workloads' ('' = none)")
    ap.add_argument("--hadamard", action="store_true",
                    help="rotate Q and K by the Hadamard transform in the timed prepass (H128; H128 + H64 for "
                         "Dqk 192); the rotated prepass is timed beside the plain one in any case")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.workload in synth.VARLEN_WORKLOADS:
        wl = varlen_workload(args.workload, args.seed)
        if args.impl == "reference":
            return run_reference(args, wl)
        return run_varlen(args, wl)
    wl = dict(synth.WORKLOADS[args.workload])
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_ours(args, wl)


def config_for(args, wl, world):
    """The line's config, the same for both arms."""
    if "lens" in wl:
        return {"workload": args.workload, "nseq": len(wl["lens"]), "tokens": wl["cu"][-1], "Hq": wl["Hq"],
                "Hkv": wl["Hkv"], "Dqk": wl["Dqk"], "Dv": wl["Dv"],
                "inputs": wl["kind"] + ", seeded, bf16 in HBM, packed [T, H, D]",
                "lengths": f"{wl['nseq']} log-uniform in [{wl['lo']}, {wl['hi']}] per rank",
                "global_batch": len(wl["lens"]) * world, "seq_len": max(wl["lens"]),
                "step": "quantize Q,K,V per (sequence, head) + FP8 Lean-P causal attention, packed batch",
                "l2": "flushed before every timed step (256 MiB write, untimed)",
                "parallelism": f"dp{world} (a packed batch of {world} x {len(wl['lens'])} sequences split "
                               f"into runs of sequences, one per rank; no collective)"}
    return {"workload": args.workload, "B": wl["B"], "S": wl["S"], "Hq": wl["Hq"], "Hkv": wl["Hkv"],
            "Dqk": wl["Dqk"], "Dv": wl["Dv"], "inputs": wl["kind"] + ", seeded, bf16 in HBM",
            "global_batch": wl["B"] * world, "seq_len": wl["S"],
            "step": "quantize Q,K,V (bf16 -> e4m3, per-head scale" + (", Hadamard Q/K" if args.hadamard else "")
                    + ") + FP8 Lean-P causal attention",
            "l2": "flushed before every timed step (256 MiB write, untimed)",
            "parallelism": f"dp{world} (one problem of {world} x {wl['B']} batch entries split into runs of "
                           f"(batch, kv head) slots, one per rank; no collective)"}


def _dist_setup(n):
    import torch
    import torch.distributed as dist
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def run_reference(args, wl):
    """The reference arm: the CPU oracle (plain C, fp64 attention on the
    dequantized e4m3 inputs), on a bounded sample of query rows per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from oracle import oracle as orc
    B, S, Hq, Hkv, Dqk, Dv = wl["B"], wl["S"], wl["Hq"], wl["Hkv"], wl["Dqk"], wl["Dv"]
    q, k, v = synth.make_qkv(args.seed, B, S, Hq, Hkv, Dqk, Dv, wl["kind"])
    import torch
    bf = lambda x: torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    codes = oracle_inputs(wl, args.seed, bf(q), bf(k), bf(v))
    (qc, qs), (kc, ks), (vc, vs) = codes
    deq = (orc.dequantize(qc, qs), orc.dequantize(kc, ks), orc.dequantize(vc, vs))
    # size each step so the whole run stays within about two minutes
    budget = min(2.0, 120.0 / (args.steps + args.warmup))
    probe = sample_rows(S, 8)
    t0 = time.perf_counter(); orc.attention(*deq, rows=probe); tp = time.perf_counter() - t0
    rate = row_flops(probe, Hq, Dqk, Dv, B) / max(tp, 1e-6)
    avg_row = row_flops(sample_rows(S, 64), Hq, Dqk, Dv, B) / 64
    n_rows = int(max(1, min(S, budget * rate / max(avg_row, 1.0))))
    rows = sample_rows(S, n_rows)
    fl = row_flops(rows, Hq, Dqk, Dv, B)
    for _ in range(args.warmup):
        orc.attention(*deq, rows=rows[:1])
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        orc.attention(*deq, rows=rows)
        times.append(time.perf_counter() - t0)
    tot = sum(times)
    val = fl * args.steps / tot / 1e12
    line = {"impl": "reference", "metric": METRIC_VARLEN if "lens" in wl else METRIC, "value": val,
            "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config_for(args, wl, args.gpus),
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": orc.num_threads(), "kind": "oracle",
                             "sample": f"{len(rows)} query rows x {B * Hq} heads per step (rows 0, S-1, tile "
                                       f"edges, seeded random), fp64 attention on the dequantized e4m3 inputs"
                                       + (" of the longest sequence" if "lens" in wl else "")},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ----------------------------------------------------------------- device-side legs

def _bus_id(torch, dev):
    props = torch.cuda.get_device_properties(dev)
    if all(hasattr(props, a) for a in ("pci_domain_id", "pci_bus_id", "pci_device_id")):
        return f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
    return None


def measure_gemm_peaks(torch, dev, bus, seconds):
    """cuBLAS dense GEMM throughput on this GPU, 8192^3: bf16 (torch.matmul) and
    e4m3 (torch._scaled_mm, bf16 out).  Burst: the best of 5 bursts of 10
    back-to-back launches; sustained: back to back for `seconds` with clock and
    power sampled.  Both bursts run before either sustained loop, so that no
    burst is timed on a GPU still held at its power cap by the loop before it.
    These are the denominators of the roofline fractions."""
    N = 8192
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    a = torch.randn(N, N, device=dev, generator=g).to(torch.bfloat16)
    b = torch.randn(N, N, device=dev, generator=g).to(torch.bfloat16)
    a8 = a.to(torch.float8_e4m3fn)
    b8 = b.to(torch.float8_e4m3fn).t()          # the second operand column-major
    one = torch.ones((), device=dev)
    fl = 2.0 * N ** 3
    out = {}
    gemms = (("bf16", lambda: torch.matmul(a, b)),
             ("fp8_e4m3", lambda: torch._scaled_mm(a8, b8, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)))
    for name, fn in gemms:
        for _ in range(5):
            fn()
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(5):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(10):
                fn()
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1) / 10)
        out[name] = {"burst_tflops": fl / (best * 1e-3) / 1e12, "burst_ms": best}
    for name, fn in gemms:
        entry = out[name]
        best = entry.pop("burst_ms")
        if seconds > 0:
            n = max(10, int(seconds / (best * 1e-3)))
            smp = make_sampler(bus)
            smp.start()
            time.sleep(0.1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(n):
                fn()
            e1.record()
            torch.cuda.synchronize()
            c = smp.stop() or {}
            entry.update({"sustained_tflops": fl / (e0.elapsed_time(e1) / n * 1e-3) / 1e12, "launches": n,
                          "sm_mhz": c.get("sm_mhz"), "power_w_median": c.get("power_w_median"),
                          "reasons": c.get("reasons")})
        out[name] = entry
    del a, b, a8, b8
    torch.cuda.empty_cache()
    return out


def sustained_leg(torch, fn, flops, seconds, bus):
    """One kernel back to back for about `seconds` (inputs stay where they are,
    no L2 flush) under clock / power sampling."""
    fn()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    fn()
    torch.cuda.synchronize()
    n = max(3, int(seconds / max(time.perf_counter() - t0, 1e-4)))
    smp = make_sampler(bus)
    smp.start()
    time.sleep(0.1)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n):
        fn()
    e1.record()
    torch.cuda.synchronize()
    c = smp.stop() or {}
    ms = e0.elapsed_time(e1) / n
    tf = flops / (ms * 1e-3) / 1e12
    w = c.get("power_w_median")
    return {"launches": n, "seconds": ms * n * 1e-3, "ms": ms, "tflops": tf, "sm_mhz": c.get("sm_mhz"),
            "power_w_median": w, "reasons": c.get("reasons"), "samples": c.get("samples"),
            "tflop_per_joule": (tf / w) if w else None}


def timed_steps(torch, fns, steps, flush, stream):
    """Per step: flush L2 (untimed), then events around each fn on the stream."""
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(fns) + 1)] for _ in range(steps)]
    for s in range(steps):
        flush.zero_()
        ev[s][0].record(stream)
        for i, f in enumerate(fns):
            f()
            ev[s][i + 1].record(stream)
    torch.cuda.synchronize()
    return [[ev[s][i].elapsed_time(ev[s][i + 1]) for i in range(len(fns))] for s in range(steps)]


def prepass_bytes(B, S, Hq, Hkv, Dqk, Dv, in_bytes=2):
    """Algorithmic HBM bytes of the two-pass prepass: each input read twice
    (amax pass, codes pass), one byte of code written per element."""
    n = B * S * (Hq * Dqk + Hkv * (Dqk + Dv))
    return 2 * n * in_bytes + n


def attn_bytes(B, S, Hq, Hkv, Dqk, Dv, el):
    """Algorithmic HBM bytes of one attention launch: Q, K, V read once, O (bf16) written once."""
    return B * S * (Hq * Dqk + Hkv * (Dqk + Dv)) * el + B * S * Hq * Dv * 2


class Peaks:
    """The roofline denominators: burst (a kernel timed alone, briefly) and
    sustained (a kernel timed back to back for seconds), each the larger of the
    measured (or fallback) figure and the GEMM measured in this run; FP8
    without a measurement: the bf16 figure x the nominal ratio 2."""

    def __init__(self, file_peaks, src, gemm):
        self.hbm = file_peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        bf_b = file_peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        bf_s = file_peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
        g_bf, g_f8 = (gemm or {}).get("bf16", {}), (gemm or {}).get("fp8_e4m3", {})
        self.bf16 = max(bf_b, g_bf.get("burst_tflops", 0.0))
        self.bf16_sus = max(bf_s, g_bf.get("sustained_tflops", 0.0))
        self.fp8 = max(FP8_PER_BF16 * bf_b, g_f8.get("burst_tflops", 0.0))
        self.fp8_sus = max(FP8_PER_BF16 * bf_s, g_f8.get("sustained_tflops", 0.0))
        self.source = (f"{src} file: bf16 {bf_b} burst / {bf_s} sustained (FP8 = x2); "
                       + ("cuBLAS GEMMs measured in this run; each denominator is the larger" if gemm else
                          "no GEMM measured in this run"))

    def of(self, dtype, sustained=False):
        if dtype == "fp8":
            return self.fp8_sus if sustained else self.fp8
        return self.bf16_sus if sustained else self.bf16


def roofline(achieved, peaks, dtype, kernel, sm_mhz=None, traffic=None):
    pk = peaks.of(dtype)
    r = {"bound": "tensor", "achieved": achieved, "peak": pk, "unit": "TFLOP/s", "frac": achieved / pk,
         "traffic": traffic, "kernel": kernel, "peak_kind": "burst (short timed region)",
         "peak_source": peaks.source, "frac_of_datasheet": achieved / DATASHEET[dtype]}
    if sm_mhz:
        r["frac_of_clock_scaled"] = achieved / (FLOP_PER_CLK_SM[dtype] * SMS * sm_mhz * 1e6 / 1e12)
        r["clock_scaled_at_mhz"] = sm_mhz
    return r


class FixedCase:
    """One fixed-length workload on this rank: its share of the global problem
    (batch entries rank*B .. rank*B+B-1 of world*B), the prepass and attention
    calls on resident bf16 inputs, and their outputs."""

    def __init__(self, torch, zyfa, wl, seed, rank, world, dev, hadamard):
        self.wl = wl
        B, S, Hq, Hkv, Dqk, Dv = wl["B"], wl["S"], wl["Hq"], wl["Hkv"], wl["Dqk"], wl["Dv"]
        # the rank's slots are whole batch entries of the global problem
        runs = shard.rank_slices(B * world, Hkv, world, rank)
        assert runs[0] == (rank * B, 0, Hkv) and all(r[1:] == (0, Hkv) for r in runs) and len(runs) == B
        self.q, self.k, self.v = synth.make_qkv(seed, B * world, S, Hq, Hkv, Dqk, Dv, wl["kind"], b0=rank * B, nb=B)
        self.qb, self.kb, self.vb = (torch.from_numpy(x).to(torch.bfloat16) for x in (self.q, self.k, self.v))
        self.dq, self.dk, self.dv = (t.to(dev) for t in (self.qb, self.kb, self.vb))
        u8 = lambda t: torch.empty(t.shape, dtype=torch.uint8, device=dev)
        self.cq, self.ck, self.cv = u8(self.dq), u8(self.dk), u8(self.dv)
        self.sq = torch.empty((B, Hq), dtype=torch.float32, device=dev)
        self.sk = torch.empty((B, Hkv), dtype=torch.float32, device=dev)
        self.sv = torch.empty((B, Hkv), dtype=torch.float32, device=dev)
        self.o8 = torch.empty((B, S, Hq, Dv), dtype=torch.bfloat16, device=dev)
        self.ob = torch.empty_like(self.o8)
        self.ox = torch.empty_like(self.o8)
        self.zyfa, self.had = zyfa, hadamard
        self.flops = synth.causal_flops(B, S, Hq, Dqk, Dv)

    def prepass(self, hadamard=None):
        h = self.had if hadamard is None else hadamard
        self.zyfa.quantize_qkv(self.dq, self.dk, self.dv, hadamard_qk=h,
                               out=((self.cq, self.sq), (self.ck, self.sk), (self.cv, self.sv)))

    def attn8(self):
        self.zyfa.attn_fwd(self.cq, self.ck, self.cv, o=self.o8, q_scale=self.sq, k_scale=self.sk, v_scale=self.sv)

    def attn8x(self):
        self.zyfa.attn_fwd(self.cq, self.ck, self.cv, o=self.ox, q_scale=self.sq, k_scale=self.sk, v_scale=self.sv,
                           exact_p=True)

    def attnb(self):
        self.zyfa.attn_fwd(self.dq, self.dk, self.dv, o=self.ob)

    def parity(self, seed, nrows, exact_p, hadamard):
        """Sampled rows of the outputs against the oracle (N = 1 only)."""
        from oracle import oracle as orc
        wl = self.wl
        S = wl["S"]
        bfv = lambda t: t.float().numpy()
        codes = oracle_inputs(wl, seed, bfv(self.qb), bfv(self.kb), bfv(self.vb), hadamard=hadamard)
        gpu = ((self.cq, self.sq), (self.ck, self.sk), (self.cv, self.sv))
        codes_equal = all(np.array_equal(g.cpu().numpy(), c) and np.array_equal(gs.cpu().numpy().view(np.uint32),
                                                                                   cs.view(np.uint32))
                          for (g, gs), (c, cs) in zip(gpu, codes))
        rows = sample_rows(S, nrows)
        o_ref, dt, cores, deq = time_oracle_rows(wl, codes, rows)
        o_gpu = self.o8.float().cpu().numpy()[:, rows].astype(np.float64)
        ob_ref = orc.attention(*(t.double().numpy() for t in (self.qb, self.kb, self.vb)), rows=rows)
        ob_gpu = self.ob.float().cpu().numpy()[:, rows].astype(np.float64)
        unq = orc.attention(self.q, self.k, self.v, rows=rows)
        par = {"rows_sampled": int(len(rows)), "fp8_vs_fp64_dequantized": orc.rel_fro(o_gpu, o_ref),
               "fp8_vs_fp64_unquantized": orc.rel_fro(o_gpu, unq), "bf16_vs_fp64": orc.rel_fro(ob_gpu, ob_ref),
               "fp8_vs_fp64_dequantized_worst_head": max_head_rel_fro(o_gpu, o_ref),
               "bf16_vs_fp64_worst_head": max_head_rel_fro(ob_gpu, ob_ref),
               "prepass_codes_bit_exact": bool(codes_equal), "tolerances": {"bf16": 5e-3, "fp8": 3e-2}}
        if exact_p:
            ox = self.ox.float().cpu().numpy()[:, rows].astype(np.float64)
            par["exact_p_fp8_vs_fp64_dequantized"] = orc.rel_fro(ox, o_ref)
            par["exact_p_fp8_vs_fp64_unquantized"] = orc.rel_fro(ox, unq)
        bad = [k2 for k2, tol in (("fp8_vs_fp64_dequantized", 3e-2), ("bf16_vs_fp64", 5e-3),
                                  ("exact_p_fp8_vs_fp64_dequantized", 3e-2))
               if k2 in par and not par[k2] <= tol] + ([] if codes_equal else ["prepass_codes_bit_exact"])
        return par, bad, (rows, dt, cores, deq)

    def free(self):
        for n in ("dq", "dk", "dv", "cq", "ck", "cv", "sq", "sk", "sv", "o8", "ob", "ox"):
            setattr(self, n, None)


def run_fixed_timing(torch, case, steps, warmup, flush, stream, exact_p, barrier):
    """Warm-up, then the timed regions: FP8 step (prepass + attention), BF16
    attention, the exact-P ablation, the rotated prepass.  ms per launch each."""
    for _ in range(warmup):
        case.prepass(); case.attn8(); case.attnb()
        if exact_p:
            case.attn8x()
    barrier()
    per8 = timed_steps(torch, [case.prepass, case.attn8], steps, flush, stream)
    barrier()
    perb = timed_steps(torch, [case.attnb], steps, flush, stream)
    barrier()
    t = {"step": sum(a + b for a, b in per8) / steps, "attn8": sum(b for _, b in per8) / steps,
         "prepass": sum(a for a, _ in per8) / steps, "bf16": sum(x[0] for x in perb) / steps}
    if exact_p:
        perx = timed_steps(torch, [case.attn8x], steps, flush, stream)
        t["exact_p"] = sum(x[0] for x in perx) / steps
        barrier()
    # the rotated prepass (Hadamard on Q and K), restored to the timed mode after
    other = not case.had
    perh = timed_steps(torch, [lambda: case.prepass(other)], max(3, steps // 2), flush, stream)
    t["prepass_hadamard" if other else "prepass_plain"] = sum(x[0] for x in perh) / len(perh)
    case.prepass()
    case.attn8(); case.attnb()
    if exact_p:
        case.attn8x()
    torch.cuda.synchronize()
    barrier()
    return t


def run_ours(args, wl):
    import torch
    import torch.distributed as dist

    from bf16_causal_prefill_fp8_b200 import zyfa

    rank, world, local = _dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    B, S, Hq, Hkv, Dqk, Dv = wl["B"], wl["S"], wl["Hq"], wl["Hkv"], wl["Dqk"], wl["Dv"]
    file_peaks, peak_src = load_peaks()
    bus = _bus_id(torch, dev)
    stream = torch.cuda.current_stream()
    exact_p = not args.no_exact_p

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    mx = lambda x: shard.max_over_ranks(x, device=dev)
    gemm = measure_gemm_peaks(torch, dev, bus, args.peaks) if args.peaks > 0 else None
    peaks = Peaks(file_peaks, peak_src, gemm)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    case = FixedCase(torch, zyfa, wl, args.seed, rank, world, dev, args.hadamard)
    flops = case.flops
    for _ in range(args.warmup):
        case.prepass(); case.attn8(); case.attnb()
    barrier()
    if zyfa.device_status() != zyfa.OK:
        raise RuntimeError("device wait timeout during warm-up")

    # the headline timed region: FP8 steps, then BF16 attention, under sampling
    clocks = make_sampler(bus) if rank == 0 and bus else None
    if clocks:
        clocks.start()
        time.sleep(0.1)
    barrier()
    per8 = timed_steps(torch, [case.prepass, case.attn8], args.steps, flush, stream)
    barrier()
    perb = timed_steps(torch, [case.attnb], args.steps, flush, stream)
    barrier()
    clk = clocks.stop() if clocks else None
    if zyfa.device_status() != zyfa.OK:
        raise RuntimeError("device wait timeout in the timed region")
    ms8 = mx(sum(a + b for a, b in per8) / args.steps)
    ms8_attn = mx(sum(b for _, b in per8) / args.steps)
    ms8_pre = mx(sum(a for a, _ in per8) / args.steps)
    msb = mx(sum(x[0] for x in perb) / args.steps)

    # exact-P ablation and the rotated (or plain) prepass, same timing rules
    msx = None
    if exact_p:
        for _ in range(args.warmup):
            case.attn8x()
        barrier()
        perx = timed_steps(torch, [case.attn8x], args.steps, flush, stream)
        barrier()
        msx = mx(sum(x[0] for x in perx) / args.steps)
    other = not args.hadamard
    perh = timed_steps(torch, [lambda: case.prepass(other)], max(3, args.steps // 2), flush, stream)
    ms_pre_other = mx(sum(x[0] for x in perh) / len(perh))
    case.prepass()                      # the timed mode's codes again, for parity
    case.attn8()
    barrier()
    if zyfa.device_status() != zyfa.OK:
        raise RuntimeError("device wait timeout in the ablation or prepass legs")

    # sustained leg: each kernel back to back for seconds (rank 0 samples; all ranks run)
    sus = None
    if args.sustained > 0:
        sus = {}
        legs = [("fp8_lean_p", case.attn8)] + ([("fp8_exact_p", case.attn8x)] if exact_p else []) + \
               [("bf16", case.attnb)]
        for name, fn in legs:
            barrier()
            r = sustained_leg(torch, fn, flops, args.sustained, bus) if bus else None
            if r:
                dt = "bf16" if name == "bf16" else "fp8"
                r["peak"] = peaks.of(dt, sustained=True)
                r["frac"] = r["tflops"] / r["peak"]
                r["frac_of_clock_scaled"] = (r["tflops"] / (FLOP_PER_CLK_SM[dt] * SMS * r["sm_mhz"] * 1e6 / 1e12)
                                             if r.get("sm_mhz") else None)
            sus[name] = r
        barrier()
        if zyfa.device_status() != zyfa.OK:
            raise RuntimeError("device wait timeout in the sustained leg")

    value = world * flops / (ms8 * 1e-3) / 1e12
    value_b = world * flops / (msb * 1e-3) / 1e12
    ach8 = flops / (ms8_attn * 1e-3) / 1e12
    achb = flops / (msb * 1e-3) / 1e12
    sm_mhz = clk.get("sm_mhz") if clk else None

    # e2e: the same FP8 step through the public API with host buffers
    pin = [t.pin_memory() for t in (case.qb, case.kb, case.vb)]
    host_o = torch.empty(case.o8.shape, dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        case.dq.copy_(pin[0], non_blocking=True); case.dk.copy_(pin[1], non_blocking=True)
        case.dv.copy_(pin[2], non_blocking=True)
        case.prepass(); case.attn8()
        host_o.copy_(case.o8, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e_serial = mx(e0.elapsed_time(e1) / e2e_steps)
    h2d = sum(t.numel() * t.element_size() for t in pin)
    d2h = host_o.numel() * host_o.element_size()
    ref_o = case.o8.cpu()
    ms_pipe, pipe_note = float("inf"), None
    try:
        bufs = [(case.dq, case.dk, case.dv), tuple(torch.empty_like(t) for t in (case.dq, case.dk, case.dv))]
        outs = [torch.empty_like(case.o8), torch.empty_like(case.o8)]
        host_outs = [host_o, torch.empty(case.o8.shape, dtype=torch.bfloat16).pin_memory()]

        def step_on(sidx):
            xq, xk, xv = bufs[sidx]
            zyfa.quantize_qkv(xq, xk, xv, hadamard_qk=args.hadamard,
                              out=((case.cq, case.sq), (case.ck, case.sk), (case.cv, case.sv)))
            zyfa.attn_fwd(case.cq, case.ck, case.cv, o=outs[sidx], q_scale=case.sq, k_scale=case.sk,
                          v_scale=case.sv)

        barrier()
        ms_try = e2e_pipelined(torch, pin, bufs, step_on, outs, host_outs, e2e_steps)
        if torch.equal(host_outs[(e2e_steps - 1) % 2], ref_o):
            ms_pipe = ms_try
        else:
            pipe_note = "pipelined output differs from the resident-input output"
        del bufs, outs
    except Exception as exc:   # the serial figure stands; say why
        pipe_note = f"pipelined e2e failed: {exc!r}"[:200]
        torch.cuda.synchronize()
    ms_pipe = mx(ms_pipe)
    ms_e2e = ms_pipe if ms_pipe != float("inf") else ms_e2e_serial
    case.prepass(); case.attn8()
    torch.cuda.synchronize()

    # sampled full-size parity + CPU baseline (rank 0, N = 1 only)
    parity, cpu = None, None
    if world == 1:
        parity, bad, (rows, dt, cores, deq_codes) = case.parity(args.seed, 96 if S >= 8192 else 256, exact_p,
                                                                args.hadamard)
        if bad:
            # a throughput number from a kernel that fails parity is not a measurement
            print(f"bench: parity failed ({', '.join(bad)}): {json.dumps(parity)}", file=sys.stderr)
            return 1
        cpu_val, cpu_rows, cpu_dt = time_oracle_baseline(deq_codes, S, rows, dt, Hq, Dqk, Dv, B)
        cpu = {"value": cpu_val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": f"{cpu_rows} query rows x {B * Hq} heads (rows 0, S-1, tile edges, seeded random) of "
                         f"{args.workload}: fp64 causal attention on the dequantized e4m3 inputs, {cpu_dt:.1f} s"}

    # the pages' other shapes, each at N GPUs like the headline
    subs = {}
    extra = [w for w in (args.also or "").split(",") if w and w != args.workload]
    if extra:
        case.free()
        del pin, host_o
        torch.cuda.empty_cache()
        for wname in extra:
            subs[wname] = run_extra(torch, zyfa, args, wname, rank, world, dev, flush, stream, peaks, barrier, mx,
                                    bus)
            if subs[wname].get("parity_failed"):
                print(f"bench: parity failed on {wname}: {json.dumps(subs[wname].get('parity'))}", file=sys.stderr)
                return 1
            torch.cuda.empty_cache()

    if rank != 0:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    pre_bytes = prepass_bytes(B, S, Hq, Hkv, Dqk, Dv)
    ms_had = ms_pre_other if not args.hadamard else ms8_pre
    ms_plain = ms8_pre if not args.hadamard else ms_pre_other
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms8, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8e4m3", "data": "synthetic",
        "config": config_for(args, wl, world),
        "roofline": roofline(ach8, peaks, "fp8", fp8_kernel_name(Dqk), sm_mhz, load_traffic(args.workload)),
        "bf16": {"value": value_b, "unit": "TFLOP/s", "ms_per_step": msb,
                 "roofline": roofline(achb, peaks, "bf16", f"attn_fwd_kernel<BF16,{Dqk}>", sm_mhz)},
        "fp8_breakdown_ms": {"prepass": ms8_pre, "attention": ms8_attn},
        "prepass": {"ms": ms8_pre, "bytes": pre_bytes, "achieved_gbs": pre_bytes / (ms8_pre * 1e-3) / 1e9,
                    "peak_gbs": peaks.hbm, "frac": pre_bytes / (ms8_pre * 1e-3) / 1e9 / peaks.hbm,
                    "bytes_rule": "inputs read twice (amax pass, codes pass) + 1 byte of code per element",
                    "hadamard_ms": ms_had, "plain_ms": ms_plain,
                    "hadamard_extra_share_of_attention": (ms_had - ms_plain) / ms8_attn},
        "peaks_measured": gemm,
        "sustained": sus,
        "ablation": None if msx is None else {
            "exact_p": {"kernel": fp8_kernel_name(Dqk, "exact P"), "attention_ms": msx,
                        "attention_tflops": flops / (msx * 1e-3) / 1e12,
                        "frac": flops / (msx * 1e-3) / 1e12 / peaks.fp8,
                        "lean_p_attention_tflops": ach8,
                        "note": "same codes, scales, deferred max, block shift and row sum; P = e4m3(ex2(.)) "
                                "instead of Lean P; errors under parity.exact_p_*"}},
        "workloads": subs or None,
        "e2e": {"value": world * flops / (ms_e2e * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
                "serial_ms_per_step": ms_e2e_serial,
                "pipelined": ms_pipe != float("inf"), "note": pipe_note,
                "path": "pinned host bf16 Q,K,V -> H2D -> zyfa_quantize_qkv -> zyfa_attn_fwd -> D2H O; "
                        "pipelined: each step's H2D overlaps the previous step's compute and its D2H the "
                        "next step's (copy and D2H streams, two buffer sets)"},
        "gpu_launches": args.steps * (4 + 1 + 1),
        "clocks": clk,
        "parity": parity,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_extra(torch, zyfa, args, wname, rank, world, dev, flush, stream, peaks, barrier, mx, bus=None):
    """One of the further workloads: timed like the headline (fewer steps),
    with its roofline and sampled parity; a fixed-length one also gets short
    sustained legs of both FP8 kernels (Lean P and exact P) for the energy and
    clock comparison across input kinds."""
    steps = max(3, min(args.steps, 10))
    if wname in synth.VARLEN_WORKLOADS:
        wl = varlen_workload(wname, args.seed)
        vc = VarlenCase(torch, zyfa, wl, args.seed, rank, world, dev)
        t = vc.timing(steps, args.warmup, flush, stream, barrier)
        out = {k2: mx(v) for k2, v in t.items()}
        res = {"kind": "packed batch", "nseq": len(vc.lens), "tokens": vc.T, "flops": vc.flops,
               "fp8_step_tflops": world * vc.flops / (out["step"] * 1e-3) / 1e12,
               "fp8_attention_tflops": vc.flops / (out["attn8"] * 1e-3) / 1e12,
               "bf16_attention_tflops": vc.flops / (out["bf16"] * 1e-3) / 1e12, "ms": out,
               "roofline": {"fp8": roofline(vc.flops / (out["attn8"] * 1e-3) / 1e12, peaks, "fp8",
                                            fp8_kernel_name(wl['Dqk'], "varlen")),
                            "bf16": roofline(vc.flops / (out["bf16"] * 1e-3) / 1e12, peaks, "bf16",
                                             f"attn_fwd_kernel<BF16,{wl['Dqk']},varlen>")}}
        if world == 1:
            par, bad = vc.parity()
            res["parity"] = par
            res["parity_failed"] = bool(bad)
        vc.free()
        return res
    wl = dict(synth.WORKLOADS[wname])
    case = FixedCase(torch, zyfa, wl, args.seed, rank, world, dev, False)
    t = run_fixed_timing(torch, case, steps, args.warmup, flush, stream, True, barrier)
    out = {k2: mx(v) for k2, v in t.items()}
    fl = case.flops
    Dqk = wl["Dqk"]
    res = {"B": wl["B"], "S": wl["S"], "Hq": wl["Hq"], "Hkv": wl["Hkv"], "Dqk": Dqk, "Dv": wl["Dv"],
           "inputs": wl["kind"], "flops": fl, "steps": steps,
           "fp8_step_tflops": world * fl / (out["step"] * 1e-3) / 1e12,
           "fp8_attention_tflops": fl / (out["attn8"] * 1e-3) / 1e12,
           "bf16_attention_tflops": fl / (out["bf16"] * 1e-3) / 1e12,
           "exact_p_attention_tflops": fl / (out["exact_p"] * 1e-3) / 1e12, "ms": out,
           "prepass_gbs": prepass_bytes(wl["B"], wl["S"], wl["Hq"], wl["Hkv"], Dqk, wl["Dv"]) / (out["prepass"] * 1e-3) / 1e9,
           "roofline": {"fp8": roofline(fl / (out["attn8"] * 1e-3) / 1e12, peaks, "fp8", fp8_kernel_name(Dqk)),
                        "bf16": roofline(fl / (out["bf16"] * 1e-3) / 1e12, peaks, "bf16",
                                         f"attn_fwd_kernel<BF16,{Dqk}>")}}
    if args.sustained > 0:
        sus = {}
        for name, fn in (("fp8_lean_p", case.attn8), ("fp8_exact_p", case.attn8x)):
            barrier()
            r = sustained_leg(torch, fn, fl, min(args.sustained, 1.0), bus) if bus else None
            if r:
                r["peak"] = peaks.of("fp8", sustained=True)
                r["frac"] = r["tflops"] / r["peak"]
            sus[name] = r
        barrier()
        res["sustained"] = sus
    if world == 1:
        par, bad, _ = case.parity(args.seed, 24, True, False)
        res["parity"] = par
        res["parity_failed"] = bool(bad)
    case.free()
    return res


# ----------------------------------------------------------------- packed batches

METRIC_VARLEN = "causal prefill attn TFLOP/s, packed variable-length batch (FP8 e4m3 & BF16, D=128)"


def varlen_workload(name, seed):
    """The packed workload: its lengths and offsets, and (for the reference arm
    and the CPU baseline) the longest sequence as a one-sequence workload."""
    wl = dict(synth.VARLEN_WORKLOADS[name])
    lens = synth.varlen_lengths(seed, wl["nseq"], wl["lo"], wl["hi"])
    wl["lens"] = lens
    wl["cu"] = [0] + [int(x) for x in np.cumsum(lens)]
    wl["B"], wl["S"] = 1, max(lens)
    return wl


def varlen_flops(lens, Hq, Dqk, Dv):
    return sum(synth.causal_flops(1, n, Hq, Dqk, Dv) for n in lens)


def varlen_parity_sequences(lens):
    """Indices of the sequences the sampled parity check covers: the longest,
    the shortest non-empty one and the median."""
    order = sorted((n, s) for s, n in enumerate(lens) if n > 0)
    pick = [order[-1][1], order[0][1], order[len(order) // 2][1]]
    return sorted(set(pick))


class VarlenCase:
    """The packed workload on this rank: sequences rank*n .. rank*n+n-1 of a
    global batch of world*n (lengths drawn for the whole batch), packed back to
    back, with the varlen prepass and attention calls."""

    def __init__(self, torch, zyfa, wl, seed, rank, world, dev):
        self.wl, self.zyfa = wl, zyfa
        n = wl["nseq"]
        glens = synth.varlen_lengths(seed, n * world, wl["lo"], wl["hi"])
        gcu = [0] + [int(x) for x in np.cumsum(glens)]
        self.lens = glens[rank * n:(rank + 1) * n]
        r0, r1 = gcu[rank * n], gcu[(rank + 1) * n]
        self.cu = [c - r0 for c in gcu[rank * n:(rank + 1) * n + 1]]
        self.T = r1 - r0
        Hq, Hkv, Dqk, Dv = wl["Hq"], wl["Hkv"], wl["Dqk"], wl["Dv"]
        # rows r0 .. r1-1 of the global packed tensors [1, T_global, H, D]
        q, k, v = synth.make_qkv_rows(seed, gcu[-1], Hq, Hkv, Dqk, Dv, wl["kind"], r0, r1)
        self.q, self.k, self.v = q, k, v
        self.qb, self.kb, self.vb = (torch.from_numpy(x).to(torch.bfloat16) for x in (q, k, v))
        self.dq, self.dk, self.dv = (t.to(dev) for t in (self.qb, self.kb, self.vb))
        u8 = lambda t: torch.empty(t.shape, dtype=torch.uint8, device=dev)
        self.cq, self.ck, self.cv = u8(self.dq), u8(self.dk), u8(self.dv)
        self.sq = torch.empty((n, Hq), dtype=torch.float32, device=dev)
        self.sk = torch.empty((n, Hkv), dtype=torch.float32, device=dev)
        self.sv = torch.empty((n, Hkv), dtype=torch.float32, device=dev)
        self.o8 = torch.empty((self.T, Hq, Dv), dtype=torch.bfloat16, device=dev)
        self.ob = torch.empty_like(self.o8)
        self.flops = varlen_flops(self.lens, Hq, Dqk, Dv)

    def prepass(self, hadamard=False):
        self.zyfa.quantize_qkv_varlen(self.dq, self.dk, self.dv, self.cu, hadamard_qk=hadamard,
                                      out=((self.cq, self.sq), (self.ck, self.sk), (self.cv, self.sv)))

    def attn8(self):
        self.zyfa.attn_fwd_varlen(self.cq, self.ck, self.cv, self.cu, o=self.o8, q_scale=self.sq, k_scale=self.sk,
                                  v_scale=self.sv)

    def attnb(self):
        self.zyfa.attn_fwd_varlen(self.dq, self.dk, self.dv, self.cu, o=self.ob)

    def timing(self, steps, warmup, flush, stream, barrier):
        import torch
        for _ in range(warmup):
            self.prepass(); self.attn8(); self.attnb()
        barrier()
        per8 = timed_steps(torch, [self.prepass, self.attn8], steps, flush, stream)
        barrier()
        perb = timed_steps(torch, [self.attnb], steps, flush, stream)
        barrier()
        self.prepass(); self.attn8(); self.attnb()
        torch.cuda.synchronize()
        return {"step": sum(a + b for a, b in per8) / steps, "attn8": sum(b for _, b in per8) / steps,
                "prepass": sum(a for a, _ in per8) / steps, "bf16": sum(x[0] for x in perb) / steps}

    def parity(self):
        """Sampled rows of the longest, the shortest and the median sequence
        against the oracle; the prepass codes and scales byte for byte."""
        from oracle import oracle as orc
        cu, lens = self.cu, self.lens
        xq, xk, xv = (t.float().numpy() for t in (self.qb, self.kb, self.vb))
        codes = [orc.quantize_varlen(xq, cu, False), orc.quantize_varlen(xk, cu, False),
                 orc.quantize_varlen(xv, cu, False)]
        codes_equal = all(np.array_equal(g.cpu().numpy(), c) and np.array_equal(gs.cpu().numpy(), cs)
                          for (g, gs), (c, cs) in zip(((self.cq, self.sq), (self.ck, self.sk), (self.cv, self.sv)),
                                                      codes))
        o8h, obh = self.o8.float().cpu().numpy(), self.ob.float().cpu().numpy()
        err8, errb, err_unq, rows_total = [], [], [], 0
        self.deq_long, self.t_orc = None, 0.0
        for s in varlen_parity_sequences(lens):
            r0, r1 = cu[s], cu[s + 1]
            rows = sample_rows(r1 - r0, 48)
            deq = tuple(orc.dequantize(c[None, r0:r1], sc[s:s + 1]) for c, sc in codes)
            ref = orc.attention(*deq, rows=rows)[0]
            refb = orc.attention(*(x[None, r0:r1].astype(np.float64) for x in (xq, xk, xv)), rows=rows)[0]
            unq = orc.attention(*(x[r0:r1][None] for x in (self.q, self.k, self.v)), rows=rows)[0]
            err8.append(orc.rel_fro(o8h[r0:r1][rows], ref))
            errb.append(orc.rel_fro(obh[r0:r1][rows], refb))
            err_unq.append(orc.rel_fro(o8h[r0:r1][rows], unq))
            rows_total += len(rows)
            if r1 - r0 == max(lens):
                self.deq_long = deq
        par = {"sequences_sampled": varlen_parity_sequences(lens), "rows_sampled": rows_total,
               "fp8_vs_fp64_dequantized": max(err8), "fp8_vs_fp64_unquantized": max(err_unq),
               "bf16_vs_fp64": max(errb), "prepass_codes_bit_exact": bool(codes_equal),
               "tolerances": {"bf16": 5e-3, "fp8": 3e-2}}
        bad = [k2 for k2, tol in (("fp8_vs_fp64_dequantized", 3e-2), ("bf16_vs_fp64", 5e-3))
               if not par[k2] <= tol] + ([] if codes_equal else ["prepass_codes_bit_exact"])
        return par, bad

    def free(self):
        for n in ("dq", "dk", "dv", "cq", "ck", "cv", "sq", "sk", "sv", "o8", "ob"):
            setattr(self, n, None)


def run_varlen(args, wl):
    """The packed workload as the headline line: zyfa_quantize_qkv_varlen +
    zyfa_attn_fwd_varlen (FP8) per step, the BF16 varlen attention timed
    alongside, sampled parity of three sequences against the oracle."""
    import torch
    import torch.distributed as dist

    from bf16_causal_prefill_fp8_b200 import zyfa

    rank, world, local = _dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    file_peaks, peak_src = load_peaks()
    bus = _bus_id(torch, dev)
    stream = torch.cuda.current_stream()

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    mx = lambda x: shard.max_over_ranks(x, device=dev)
    gemm = measure_gemm_peaks(torch, dev, bus, args.peaks) if args.peaks > 0 else None
    peaks = Peaks(file_peaks, peak_src, gemm)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    vc = VarlenCase(torch, zyfa, wl, args.seed, rank, world, dev)
    for _ in range(args.warmup):
        vc.prepass(); vc.attn8(); vc.attnb()
    barrier()
    clocks = make_sampler(bus) if rank == 0 and bus else None
    if clocks:
        clocks.start()
        time.sleep(0.1)
    t = vc.timing(args.steps, 1, flush, stream, barrier)
    clk = clocks.stop() if clocks else None
    if zyfa.device_status() != zyfa.OK:
        raise RuntimeError("device wait timeout in the timed region")
    ms = {k2: mx(v) for k2, v in t.items()}
    pin = [x.pin_memory() for x in (vc.qb, vc.kb, vc.vb)]
    host_o = torch.empty(vc.o8.shape, dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        vc.dq.copy_(pin[0], non_blocking=True); vc.dk.copy_(pin[1], non_blocking=True)
        vc.dv.copy_(pin[2], non_blocking=True)
        vc.prepass(); vc.attn8()
        host_o.copy_(vc.o8, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = mx(e0.elapsed_time(e1) / e2e_steps)
    vc.attnb()
    torch.cuda.synchronize()
    if rank != 0:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0
    flops = vc.flops
    ach8 = flops / (ms["attn8"] * 1e-3) / 1e12
    achb = flops / (ms["bf16"] * 1e-3) / 1e12
    sm_mhz = clk.get("sm_mhz") if clk else None
    parity, cpu = None, None
    if world == 1:
        from oracle import oracle as orc
        parity, bad = vc.parity()
        if bad:
            print(f"bench: parity failed ({', '.join(bad)}): {json.dumps(parity)}", file=sys.stderr)
            return 1
        S_long = max(vc.lens)
        rows_long = sample_rows(S_long, 48)
        t0 = time.perf_counter()
        orc.attention(*vc.deq_long, rows=rows_long)
        dt_long = time.perf_counter() - t0
        cpu_val, cpu_rows, cpu_dt = time_oracle_baseline(vc.deq_long, S_long, rows_long, dt_long, wl["Hq"],
                                                         wl["Dqk"], wl["Dv"], 1)
        cpu = {"value": cpu_val, "unit": "TFLOP/s", "cores": orc.num_threads(), "kind": "oracle",
               "sample": f"{cpu_rows} query rows x {wl['Hq']} heads of the longest sequence ({S_long} rows) of "
                         f"{args.workload}: fp64 causal attention on the dequantized e4m3 inputs, {cpu_dt:.1f} s"}
    line = {
        "metric": METRIC_VARLEN, "value": world * flops / (ms["step"] * 1e-3) / 1e12, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms["step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp8e4m3",
        "data": "synthetic", "config": dict(config_for(args, wl, world), lens=vc.lens),
        "roofline": roofline(ach8, peaks, "fp8", fp8_kernel_name(wl['Dqk'], "varlen"), sm_mhz),
        "bf16": {"value": world * flops / (ms["bf16"] * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms["bf16"],
                 "roofline": roofline(achb, peaks, "bf16", f"attn_fwd_kernel<BF16,{wl['Dqk']},varlen>", sm_mhz)},
        "fp8_breakdown_ms": {"prepass": ms["prepass"], "attention": ms["attn8"]},
        "peaks_measured": gemm,
        "e2e": {"value": world * flops / (ms_e2e * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in pin),
                "d2h_bytes_per_step": host_o.numel() * host_o.element_size(), "ms_per_step": ms_e2e,
                "path": "pinned host bf16 Q,K,V -> H2D -> zyfa_quantize_qkv_varlen -> zyfa_attn_fwd_varlen -> D2H O"},
        "gpu_launches": args.steps * (4 + 1 + 1),
        "clocks": clk,
        "parity": parity,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


KERNEL_SOURCES = ("attn_fwd.cuh", "attn_fwd_wide.cuh", "leanp.cuh", "ptx.cuh")


def fp8_kernel_name(Dqk, extra=""):
    """The FP8 attention kernel instance the library runs for Dqk: 256-key KV
    tiles for Dqk 128 (attn_fwd_wide_kernel), 128-key tiles otherwise."""
    tail = f",{extra}" if extra else ""
    if Dqk == 128:
        return f"attn_fwd_wide_kernel<FP8,128{tail}>"
    return f"attn_fwd_kernel<FP8,{Dqk}{tail}>"


def kernel_source_hash():
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, "bf16_causal_prefill_fp8_b200", "csrc", f), "rb").read())
    return h.hexdigest()


def load_traffic(workload):
    """DRAM bytes per attention launch from the committed ncu summary; null
    once the kernel sources differ from the ones the counters were taken on."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(p):
        d = json.load(open(p))
        e = d.get(workload)
        if e and e.get("source_sha256") == kernel_source_hash():
            return e.get("bytes_per_launch")
    return None


if __name__ == "__main__":
    sys.exit(main())
