"""GPU parity of the product path kda_fwd (the fused tcgen05 kernel for
lower_bound >= -9.5) against the fp64 recurrent oracle."""
import numpy as np
import pytest
import torch

import kda_workloads as W
import oracle
from kda_testutil import alloc_final, check, run_oracle, to_device

pytestmark = pytest.mark.gpu


def _kda():
    import kda_build as build
    build.build()
    import gated_delta_rule_135_b200 as kda
    return kda


def _run(kda, x, want_final=True, init_override="keep"):
    xd = to_device(x)
    fin = alloc_final(xd, want_final)
    init = xd["initial_state"] if init_override == "keep" else init_override
    out, fin = kda.kda_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"],
                           x["lower_bound"], x["scale"], init, xd["cu_seqlens"], final_state=fin,
                           batch=x["batch"])
    assert kda.kda_check_device_error() == 0
    return out, fin


SMALL = [
    ("tiny_fixed_t256_h2", W.WORKLOADS[0]),
    ("one_chunk", W.custom([64], H=1, packed=False, init="normal")),
    ("partial_chunk", W.custom([37], H=2, packed=False, init="normal")),
    ("varlen_ragged", W.custom([70, 0, 129, 64, 1, 200, 17], H=3, init="normal")),
    ("many_heads", W.custom([300], H=20, packed=False, init=None)),
    ("lb_5_3", W.custom([190], H=2, packed=False, init="normal", lower_bound=-5.3)),
    ("lb_steep_7", W.custom([190, 70], H=2, init="normal", lower_bound=-7.0)),
    ("lb_at_limit_9_5", W.custom([190], H=3, packed=False, init="normal", lower_bound=-9.5)),
    ("lb_mild", W.custom([190], H=2, packed=False, init="normal", lower_bound=-1.0)),
]


@pytest.mark.parametrize("name,w", SMALL, ids=[s[0] for s in SMALL])
def test_fused_matches_oracle(name, w):
    kda = _kda()
    x = W.make_inputs(w)
    out, fin = _run(kda, x)
    ref_o, ref_f = run_oracle(x)
    check(out, fin, ref_o, ref_f, name)


def test_fused_null_initial_equals_zero_initial_bitwise():
    kda = _kda()
    x = W.make_inputs(W.custom([150, 33], H=2, init="zero"))
    o1, f1 = _run(kda, x)
    o2, f2 = _run(kda, x, init_override=None)
    assert torch.equal(o1, o2) and torch.equal(f1, f2)


def test_fused_is_deterministic():
    kda = _kda()
    x = W.make_inputs(W.custom([500, 200], H=4, init="normal"))
    o1, f1 = _run(kda, x)
    o2, f2 = _run(kda, x)
    assert torch.equal(o1, o2) and torch.equal(f1, f2)


def test_fused_in_place_state_update():
    kda = _kda()
    x = W.make_inputs(W.custom([130, 64], H=2, init="normal"))
    xd = to_device(x)
    ref_o, ref_f = run_oracle(x)
    st = xd["initial_state"].clone()
    out, _ = kda.kda_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"],
                         x["lower_bound"], x["scale"], st, xd["cu_seqlens"], final_state=st)
    check(out, st, ref_o, ref_f, "in-place")


def test_fused_without_final_state():
    kda = _kda()
    x = W.make_inputs(W.custom([100], H=2, packed=False, init="normal"))
    out, fin = _run(kda, x, want_final=False)
    ref_o, _ = run_oracle(x)
    check(out, None, ref_o, None, "no-final")


def test_fused_split_and_resume():
    kda = _kda()
    w = W.custom([333], H=3, packed=False, init="normal")
    x = W.make_inputs(w)
    ref_o, ref_f = run_oracle(x)
    a, b = dict(x), dict(x)
    t1 = 150
    for key in ("q", "k", "v", "g", "beta"):
        a[key] = x[key][:t1]
        b[key] = x[key][t1:]
    a["seqlen"] = t1
    b["seqlen"] = w.T - t1
    oa, fa = _run(kda, a)
    b["initial_state"] = fa.cpu()
    ob, fb = _run(kda, b)
    check(torch.cat([oa, ob]), fb, ref_o, ref_f, "split/resume")


@pytest.mark.parametrize("wid", [3, 2, 1, 4])
def test_fused_full_size_workloads(wid):
    """The four large workloads compared in full against the oracle: 8 x 1024 stateful
    (H=64), T=8192 H=96 varlen, T=8192 H=64 fixed, and T=131072 H=32 with states."""
    kda = _kda()
    w = W.WORKLOADS[wid]
    x = W.make_inputs(w)
    out, fin = _run(kda, x, want_final=True)
    ref_o, ref_f = run_oracle(x)
    check(out, fin, ref_o, ref_f, w.name)
