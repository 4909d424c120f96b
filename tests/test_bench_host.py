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


class _FakeCuda:
    """Streams, events and copies as queues of operations, run in a random
    order that respects stream order and event waits, with every buffer
    tagged by the step whose data it holds: checks bench.e2e_pipelined's
    hazards without a GPU."""

    def __init__(self, rng):
        self.rng = rng
        self.streams = []
        self.cur = self.Stream()
        self.log = []

    # --- the torch.cuda surface e2e_pipelined uses
    def Stream(self):
        s = _FakeStream(self)
        self.streams.append(s)
        return s

    def Event(self, enable_timing=False):
        return _FakeEvent()

    def current_stream(self):
        return self.cur

    def stream(self, s):
        fake = self

        class _Ctx:
            def __enter__(self_):
                self_.prev = fake.cur
                fake.cur = s

            def __exit__(self_, *a):
                fake.cur = self_.prev
        return _Ctx()

    def synchronize(self):
        while any(s.q for s in self.streams):
            ready = [s for s in self.streams if s.q and s.ready()]
            assert ready, "deadlock: every stream waits"
            self.rng.choice(ready).step()


class _FakeEvent:
    def __init__(self):
        self.target = None          # (stream, op index) of the latest record

    def record(self, stream):
        self.target = stream.enqueue(("record",))

    def elapsed_time(self, other):
        return 1.0


class _FakeStream:
    def __init__(self, cuda):
        self.cuda, self.q, self.done = cuda, [], 0

    def enqueue(self, op):
        self.q.append(op)
        return (self, self.done + len(self.q) - 1)

    def wait_event(self, ev):
        if ev.target is not None:
            self.enqueue(("wait", ev.target))

    def ready(self):
        op = self.q[0]
        if op[0] != "wait":
            return True
        st, idx = op[1]
        return st.done > idx

    def step(self):
        op = self.q.pop(0)
        self.done += 1
        if op[0] == "run":
            op[1]()


class _FakeTensor:
    def __init__(self, cuda, name):
        self.cuda, self.name, self.tag, self.writes = cuda, name, None, 0

    def copy_(self, src, non_blocking=False):
        step_of_src = src.tag if isinstance(src, _FakeTensor) and src.name.startswith("out") else None
        dst = self

        def run():
            if step_of_src is not None:                    # D2H: the output must hold the step it is read for
                assert src.tag == step_of_src_expected[0], (src.name, src.tag)
            dst.tag = src.tag
        step_of_src_expected = [None]
        self.cuda.cur.enqueue(("run", run))
        return step_of_src_expected


def test_e2e_pipeline_has_no_buffer_hazards():
    import random
    for seed in range(200):
        rng = random.Random(seed)
        cuda = _FakeCuda(rng)
        fake_torch = type("T", (), {"cuda": cuda})
        steps = rng.randint(1, 7)
        pin = [_FakeTensor(cuda, f"pin{j}") for j in range(3)]
        bufs = [tuple(_FakeTensor(cuda, f"buf{s}{j}") for j in range(3)) for s in range(2)]
        outs = [_FakeTensor(cuda, f"out{s}") for s in range(2)]
        host = [_FakeTensor(cuda, f"host{s}") for s in range(2)]
        counter = {"h2d": [0, 0], "run": [0, 0], "d2h": [0, 0]}
        got = []

        for t in pin:
            t.tag = "input"

        # tag every H2D copy with its step: H2D of buffer set s happens for steps s, s + 2, ...
        orig_copy = _FakeTensor.copy_

        def copy_(self, src, non_blocking=False):
            if self.name.startswith("buf"):
                s = int(self.name[3])
                step = s + 2 * (counter["h2d"][s] // 3)
                counter["h2d"][s] += 1
                dst = self

                def run():
                    dst.tag = step
                cuda.cur.enqueue(("run", run))
            elif self.name.startswith("host"):
                s = int(self.name[4])
                step = s + 2 * counter["d2h"][s]
                counter["d2h"][s] += 1
                dst = self

                def run():
                    assert src.tag == step, f"D2H of step {step} read output of step {src.tag}"
                    dst.tag = step
                    got.append(step)
                cuda.cur.enqueue(("run", run))
            else:
                orig_copy(self, src, non_blocking)

        def run_step(s):
            step = s + 2 * counter["run"][s]
            counter["run"][s] += 1

            def run():
                for b in bufs[s]:
                    assert b.tag == step, f"compute of step {step} read {b.name} holding step {b.tag}"
                outs[s].tag = step
            cuda.cur.enqueue(("run", run))

        _FakeTensor.copy_ = copy_
        try:
            bench.e2e_pipelined(fake_torch, pin, bufs, run_step, outs, host, steps)
        finally:
            _FakeTensor.copy_ = orig_copy
        assert sorted(got) == list(range(steps))
        assert not any(s.q for s in cuda.streams)


class _GemmTorch:
    """Just enough of torch for bench.measure_gemm_peaks on the CPU: every
    GEMM call and every sustained-loop start is logged in order."""

    float8_e4m3fn = "e4m3"
    bfloat16 = "bf16"

    def __init__(self, log):
        self.log = log
        t = self

        class _Tensor:
            def to(self, dtype):
                return self

            def t(self):
                return self

        class _Event:
            def __init__(self, enable_timing=False):
                self.n = 0

            def record(self, stream=None):
                self.n = len(t.log)

            def elapsed_time(self, other):
                return 0.5 * max(1, other.n - self.n)

        class _Cuda:
            Event = _Event

            @staticmethod
            def synchronize():
                pass

            @staticmethod
            def empty_cache():
                pass

        class _Generator:
            def __init__(self, device=None):
                pass

            def manual_seed(self, s):
                return self

        self.cuda = _Cuda
        self.Generator = _Generator
        self._tensor = _Tensor

    def randn(self, *shape, device=None, generator=None):
        return self._tensor()

    def ones(self, shape, device=None):
        return self._tensor()

    def matmul(self, a, b):
        self.log.append("bf16")

    def _scaled_mm(self, a, b, scale_a=None, scale_b=None, out_dtype=None):
        self.log.append("fp8_e4m3")


def test_gemm_bursts_run_before_the_sustained_loops(monkeypatch):
    """Both burst measurements come before either sustained loop: a burst timed
    right after a seconds-long loop runs on a GPU held at its power cap."""
    log = []

    class _Sampler:
        def start(self):
            log.append("sustained")

        def stop(self):
            return {"sm_mhz": 1300, "power_w_median": 990.0, "reasons": ["sw_power_cap"]}

    monkeypatch.setattr(bench, "make_sampler", lambda bus: _Sampler())
    out = bench.measure_gemm_peaks(_GemmTorch(log), "cuda:0", None, 0.001)
    first_loop = log.index("sustained")
    bursts = log[:first_loop]
    assert "bf16" in bursts and "fp8_e4m3" in bursts
    assert log.count("sustained") == 2
    assert set(out) == {"bf16", "fp8_e4m3"}
    for entry in out.values():
        assert entry["burst_tflops"] > 0 and entry["sustained_tflops"] > 0 and "burst_ms" not in entry
