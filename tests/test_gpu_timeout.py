"""A bounded device-side wait that runs out, on purpose and without any fault.

Every kernel of the library waits on mbarriers with a wall-clock limit.  On expiry it records
KDA_DEVERR_TIMEOUT, waits for its own tensor-core work, frees its tensor memory and returns.
kda_selftest_wait_timeout walks that path: one CTA with an MMA in flight waits 1 ms on a barrier
that nothing arrives at.  The test checks the reported bit, that the MMA was drained before the
tensor memory was freed, and that the device is still usable: a normal kda_fwd right after it
matches the fp64 oracle and reports no error."""
import pytest
import torch

import kda_workloads as W
from kda_testutil import alloc_final, check, run_oracle, to_device

pytestmark = pytest.mark.gpu

KDA_DEVERR_TIMEOUT = 0x2


def _kda():
    import kda_build as build
    build.build()
    import gated_delta_rule_135_b200 as kda
    return kda


def test_bounded_wait_runs_out_and_the_device_recovers():
    kda = _kda()
    assert kda.kda_check_device_error() == 0
    observed = torch.zeros(2, dtype=torch.int32, device="cuda")
    kda.kda_selftest_wait_timeout(1_000_000, observed)      # 1 ms
    bits = kda.kda_check_device_error()
    assert bits & KDA_DEVERR_TIMEOUT, f"expected the timeout bit, got {bits:#x}"
    assert observed.tolist() == [1, 1]
    assert kda.kda_check_device_error() == 0                 # the error word was cleared

    x = W.make_inputs(W.custom([150, 70, 260], H=2, init="normal"))
    xd = to_device(x)
    fin = alloc_final(xd, True)
    out, fin = kda.kda_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"],
                           x["lower_bound"], x["scale"], xd["initial_state"], xd["cu_seqlens"], final_state=fin)
    assert kda.kda_check_device_error() == 0
    ref_o, ref_f = run_oracle(x)
    check(out, fin, ref_o, ref_f, "after the timeout")
