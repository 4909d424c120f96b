"""Failure path without a GPU fault: a bounded device wait that nothing
satisfies runs out, is reported by zyfa_device_status, and the context stays
usable."""
import pytest
import torch

from bf16_causal_prefill_fp8_b200 import zyfa

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_cleared():
    assert zyfa.device_status() == zyfa.OK
    zyfa.selftest_wait_timeout(2_000_000)          # 2 ms
    assert zyfa.device_status() == zyfa.ERR_DEVICE_TIMEOUT
    assert zyfa.device_status() == zyfa.OK         # read-and-clear
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0                # context still healthy
