"""The checked build (libzyfa_checked.so: range checks on unit indices, tile
rows, scale reads and output rows) on fixed-length and packed batches: no
check fails, and the outputs equal the normal build's bit for bit (the checks
only guard accesses).  Runs the checked library in a child process."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from bf16_causal_prefill_fp8_b200 import build, synth, zyfa

from helpers import bf16_round

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LENS = [300, 0, 1, 128, 129, 1000, 77]


def run_cases():
    """FP8 and BF16, fixed length (B 2, S 700, GQA 4/2) and packed (LENS, MLA
    shape): output bytes of every case, in order."""
    outs = []
    q, k, v = synth.make_qkv(61, 2, 700, 4, 2, 128, 128, "outlier_k")
    dq, dk, dv = (bf16_round(x).cuda() for x in (q, k, v))
    outs.append(zyfa.attn_fwd(dq, dk, dv))
    (cq, sq), (ck, sk), (cv, sv) = zyfa.quantize_qkv(dq, dk, dv)
    outs.append(zyfa.attn_fwd(cq, ck, cv, q_scale=sq, k_scale=sk, v_scale=sv))
    cu = [0] + list(np.cumsum(LENS).astype(int))
    q, k, v = synth.make_qkv(62, 1, int(sum(LENS)), 2, 2, 192, 128, "mla")
    dq, dk, dv = (bf16_round(x[0]).cuda() for x in (q, k, v))
    outs.append(zyfa.attn_fwd_varlen(dq, dk, dv, cu))
    (cq, sq), (ck, sk), (cv, sv) = zyfa.quantize_qkv_varlen(dq, dk, dv, cu, hadamard_qk=True)
    o, lse = zyfa.attn_fwd_varlen(cq, ck, cv, cu, q_scale=sq, k_scale=sk, v_scale=sv, lse=True)
    outs += [o, lse]
    torch.cuda.synchronize()
    return [t.contiguous().view(torch.uint8).cpu().numpy() for t in outs]


CHILD = r"""
import os, sys, json
sys.path.insert(0, os.path.join(sys.argv[1], "tests")); sys.path.insert(0, sys.argv[1])
import numpy as np
from bf16_causal_prefill_fp8_b200 import zyfa
assert zyfa.checked_build()
import test_gpu_z_checked_build as t
outs = t.run_cases()
np.savez(sys.argv[2], *outs)
print(json.dumps({"check": zyfa.device_check(), "status": zyfa.device_status()}))
"""


def test_checked_build_passes_its_checks_and_matches(tmp_path):
    build.build()   # both libraries (no-op when up to date)
    normal = run_cases()
    assert zyfa.device_check() == 0 and not zyfa.checked_build()
    path = str(tmp_path / "checked.npz")
    env = dict(os.environ, ZYFA_CHECKED="1")
    out = subprocess.run([sys.executable, "-c", CHILD, ROOT, path], capture_output=True, text=True, env=env,
                         timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    res = json.loads(out.stdout.strip().splitlines()[-1])
    assert res["check"] == 0 and res["status"] == zyfa.OK, res
    checked = np.load(path)
    assert len(checked.files) == len(normal)
    for i, ref in enumerate(normal):
        assert np.array_equal(checked[f"arr_{i}"], ref), i
