"""kda_fwd_staged_noalloc, the entry point for callers that cannot allocate
device memory (their memory belongs to another allocator, or allocation is
off-limits on their path): it runs the staged forward on a fixed scratch array
the library owns, so it must produce what kda_fwd_staged produces with a
caller-provided workspace.  Called through the C ABI twice in a row (the
scratch keeps the previous call's contents), and must pass both alone in a
fresh process and after the rest of the suite.

The file name sorts last so that a run stopping at the first failure has
already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import kda_workloads as W
import oracle
from kda_testutil import OUT_MAX_ABS, OUT_REL_L2, STATE_REL_L2, to_device

pytestmark = pytest.mark.gpu


def _kda():
    import kda_build as build
    build.build()
    import gated_delta_rule_135_b200 as kda
    return kda


def _noalloc_call(kda, x, xd, fin):
    """Calls the entry point through the raw C ABI (ctypes)."""
    dims = kda.make_dims(xd["q"].shape[-2], total_tokens=xd["q"].shape[0],
                         cu_seqlens=xd["cu_seqlens"], batch=x["batch"])
    out = torch.empty_like(xd["q"])
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = kda.lib().kda_fwd_staged_noalloc(
        p(xd["q"]), p(xd["k"]), p(xd["v"]), p(xd["g"]), p(xd["beta"]), p(xd["A_log"]),
        p(xd["dt_bias"]), ctypes.c_float(x["lower_bound"]), ctypes.c_float(x["scale"]),
        p(xd["initial_state"]), p(xd["cu_seqlens"]), p(out), p(fin), dims,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, kda.kda_strerror(st)
    return out


def _compare(o, f, o_ref, f_ref):
    o = o.float().cpu().numpy().astype(np.float64)
    o_ref = o_ref.float().cpu().numpy().astype(np.float64)
    assert oracle.rel_l2(o, o_ref) <= OUT_REL_L2
    assert oracle.max_abs(o, o_ref) <= OUT_MAX_ABS
    assert oracle.rel_l2(f.cpu().numpy(), f_ref.cpu().numpy()) <= STATE_REL_L2


def test_noalloc_matches_staged_twice_in_a_row():
    kda = _kda()
    cases = [W.custom([70, 0, 129, 64, 1, 200], H=3, init="normal", wid=41),
             W.custom([256], H=2, packed=False, init="zero", wid=42)]
    for w in cases:                                   # two calls in a row, different shapes
        x = W.make_inputs(w)
        xd = to_device(x)
        fin_ref = torch.empty(w.N, w.H, 128, 128, device="cuda")
        o_ref, _, _ = kda.kda_fwd_staged(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"],
                                         xd["A_log"], xd["dt_bias"], x["lower_bound"], x["scale"],
                                         xd["initial_state"], xd["cu_seqlens"],
                                         final_state=fin_ref, batch=x["batch"])
        fin = torch.full((w.N, w.H, 128, 128), float("nan"), device="cuda")
        o = _noalloc_call(kda, x, xd, fin)
        torch.cuda.synchronize()
        assert kda.kda_check_device_error() == 0
        _compare(o, fin, o_ref, fin_ref)


def test_noalloc_rejects_problems_beyond_its_scratch():
    kda = _kda()
    limit = kda.kda_noalloc_scratch_bytes()
    assert limit == 16 << 20
    w = W.custom([4096], H=4, packed=False, init=None, wid=43)      # needs ~50 MB of workspace
    x = W.make_inputs(w)
    xd = to_device(x)
    with pytest.raises(kda.KdaError) as e:
        kda.kda_fwd_staged_noalloc(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"],
                                   xd["dt_bias"], x["lower_bound"], x["scale"])
    assert e.value.status == 7
