"""Failure path on the GPU without a fault: a kernel's bounded wait runs out
(nothing ever arrives on its barrier), the status word reports it, and the
context stays usable for a normal forward right after."""

import time

import pytest
import torch

import mixture_experts_ffn_14_b200 as moe
from mixture_experts_ffn_14_b200 import workloads as W

from _harness import full_check, run_gpu

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def test_bounded_wait_times_out_and_reports():
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    t0 = time.perf_counter()
    moe.moe_selftest_bounded_wait(ws, limit_us=20_000)      # 20 ms
    st, code = moe.moe_device_status(ws)
    elapsed = time.perf_counter() - t0
    assert st == 6 and code == 0x10, (st, code)             # MOE_ERR_DEVICE_CHECK, self-test bit
    assert 0.015 < elapsed < 5.0
    # The context is still usable: a normal call right after passes parity.
    inp = W.make_torch(W.Workload("after", 100, 512, 384, dtype="bf16", seed=80), DEV)
    full_check(inp, run_gpu(inp))
