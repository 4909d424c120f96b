"""bench.py host logic without a GPU: the row sample the parity check and the
CPU baseline use, the FLOP convention, the sizing of the oracle baseline, and
the reference arm's JSON line (the oracle timed on the host cores)."""
import json
import os
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from bf16_causal_prefill_fp8_b200 import synth  # noqa: E402
from oracle import oracle as orc  # noqa: E402


def test_sample_rows_covers_edges_and_is_sorted_unique():
    for S, n in ((16384, 96), (1000, 256), (300, 96), (5, 96)):
        r = bench.sample_rows(S, n)
        assert r.dtype == np.int32 and len(r) <= min(n, S)
        assert np.all(np.diff(r) > 0) and r[0] >= 0 and r[-1] < S
        assert 0 in r and S - 1 in r
        if S > 128 and n >= 8:
            assert 127 in r and 128 in r          # a tile edge on both sides


def test_row_flops_matches_the_causal_convention():
    S, Hq, Dqk, Dv, B = 300, 4, 192, 128, 2
    full = bench.row_flops(np.arange(S), Hq, Dqk, Dv, B)
    assert full == 2.0 * B * Hq * (Dqk + Dv) * S * (S + 1) / 2
    # the headline convention 2 B Hq (S^2 / 2)(Dqk + Dv) differs only by the diagonal
    assert abs(full / (2.0 * B * Hq * (S * S / 2) * (Dqk + Dv)) - 1) < 1.0 / S + 1e-12


def test_cpu_baseline_reaches_its_time_target():
    q, k, v = synth.make_qkv(0, 1, 4096, 4, 4, 128, 128, "gaussian")
    codes = [orc.quantize(x) for x in (q, k, v)]
    rows = bench.sample_rows(4096, 96)
    old = bench.CPU_BASELINE_SECONDS
    try:
        bench.CPU_BASELINE_SECONDS = 0.5
        _, dt, cores, deq = bench.time_oracle_rows(None, codes, rows)
        tf, n_rows, secs = bench.time_oracle_baseline(deq, 4096, rows, dt, 4, 128, 128, 1)
    finally:
        bench.CPU_BASELINE_SECONDS = old
    assert cores >= 1 and tf > 0
    assert n_rows > len(rows) and 0.15 < secs < 5.0


def test_reference_arm_json_line():
    env = dict(os.environ, OMP_NUM_THREADS=os.environ.get("OMP_NUM_THREADS", "4"))
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "tiny_s512", "--steps", "2", "--warmup", "3"], capture_output=True, text=True, env=env,
                         timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["config"]["workload"] == "tiny_s512"


def test_varlen_workload_recipe():
    wl = bench.varlen_workload("varlen_gqa32x8_mix32", 0)
    lens = wl["lens"]
    assert len(lens) == wl["nseq"] == 32
    assert all(wl["lo"] <= n <= wl["hi"] for n in lens)
    assert wl["cu"][0] == 0 and wl["cu"][-1] == sum(lens)
    assert all(b - a == n for a, b, n in zip(wl["cu"], wl["cu"][1:], lens))
    assert wl["S"] == max(lens) and wl["B"] == 1
    assert bench.varlen_workload("varlen_gqa32x8_mix32", 0)["lens"] == lens      # seeded
    assert bench.varlen_workload("varlen_gqa32x8_mix32", 1)["lens"] != lens
    # FLOPs are the per-sequence causal counts summed
    assert bench.varlen_flops([512, 1000], 32, 128, 128) == (synth.causal_flops(1, 512, 32, 128, 128)
                                                              + synth.causal_flops(1, 1000, 32, 128, 128))
    picked = bench.varlen_parity_sequences([5, 0, 900, 3, 40])
    assert picked == [2, 3, 4] or picked == sorted({2, 3, 4})


def test_reference_arm_on_packed_workload():
    env = dict(os.environ, OMP_NUM_THREADS=os.environ.get("OMP_NUM_THREADS", "4"))
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "varlen_gqa32x8_mix32", "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                         env=env, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC_VARLEN and line["value"] > 0


def test_max_head_rel_fro():
    rng = np.random.default_rng(0)
    ref = rng.normal(size=(1, 5, 3, 8))
    got = ref.copy()
    got[:, :, 1, :] *= 1.01                      # head 1 off by 1 %
    assert abs(bench.max_head_rel_fro(got, ref) - 0.01) < 1e-12
    assert bench.max_head_rel_fro(ref, ref) == 0.0
    assert bench.max_head_rel_fro(got, ref) >= orc.rel_fro(got, ref)
