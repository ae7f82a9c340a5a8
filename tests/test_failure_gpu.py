"""Failure detection on the GPU: bounded waits run out, report, and leave no trace.

Every wait of the tensor-core kernels (on an mbarrier, a ready flag or a shared
counter) gives up after a time limit, counts a timeout in libkda's device status and
lets its kernel unwind. These tests shorten the limit to a millisecond and make each
kind of wait run out on a condition that never comes true, inside a small self-test
kernel that has no copy or MMA in flight; nothing here faults, traps or hangs a GPU.
They then check that the status reports it exactly once, and that a timeout nobody
has read yet does not disturb the calls that follow (each plan of the bf16 prefill
still matches the oracle).
"""
import time

import pytest
import torch

import gated_delta_rule_101_b200 as kda
import oracle
from gated_delta_rule_101_b200.inputs import prefill_inputs
from parity import check

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
LIMIT_NS = 1_000_000  # 1 ms


def _expire_all_waits():
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)  # nothing ever sets it
    result = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    kda.set_wait_limit_ns(LIMIT_NS)
    try:
        t0 = time.perf_counter()
        kda.selftest_wait_timeout(flag, result)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        kda.set_wait_limit_ns(0)
    return int(result.item()), elapsed


def test_each_kind_of_bounded_wait_runs_out_and_is_reported():
    kda.device_status()  # start from a cleared status
    bits, elapsed = _expire_all_waits()
    assert bits == 7, f"waits that gave up: {bits:03b} (mbarrier, flag, counter should all)"
    # three limits of 1 ms each, plus a launch; far below the default limit of 1 s each
    assert elapsed < 0.5, elapsed
    assert kda.device_status() == 1
    assert kda.device_status() == 0  # reading clears it


# one shape per bf16 plan (launch counts as kda_chunk_fwd_launches reports them)
PLANS = {"prep_then_chain": (1, 300, 72, 2), "fused_grid": (1, 1000, 32, 1),
         "segment_scan": (1, 3000, 2, 4)}


@pytest.mark.parametrize("plan", list(PLANS))
def test_unread_timeout_leaves_later_calls_correct(plan):
    """A timeout left unread in the status must not make later calls give up early."""
    B, T, H, launches = PLANS[plan]
    assert kda.chunk_fwd_launches(B, T, H) == launches
    bits, _ = _expire_all_waits()
    assert bits == 7
    # the status now holds an unread timeout; the default limit is back in force
    inp = prefill_inputs(B=B, T=T, H=H, dtype=torch.bfloat16, s0_std=0.1, seed=77, device=DEV)
    o, st = kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0)
    torch.cuda.synchronize()
    for h in (0, H - 1):
        sl = lambda x: x[:, :, h:h + 1]
        ro, rs = oracle.kda_fwd(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.log_alpha),
                                inp.beta[:, :, h:h + 1], inp.S0[:, h:h + 1])
        check(o[:, :, h:h + 1], ro, "bf16", f"{plan} o head {h}")
        check(st[:, h:h + 1], rs, "bf16", f"{plan} S_T head {h}")
    assert kda.device_status() == 1  # the self-test's timeouts, reported once
    assert kda.device_status() == 0
