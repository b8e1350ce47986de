"""GPU parity of kda_gdn_fwd (the scalar-gate variant: one decay per token-head) against
the fp64 oracle (gdn_recurrent: the recurrence with that decay on every channel)."""
import pytest
import torch

import kda_workloads as W
import oracle
from kda_testutil import alloc_final, check, to_device

pytestmark = pytest.mark.gpu


def _kda():
    import kda_build as build
    build.build()
    import gated_delta_rule_135_b200 as kda
    return kda


def _run(kda, x, want_final=True):
    xd = to_device(x)
    fin = alloc_final(xd, want_final)
    out, fin = kda.kda_gdn_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"],
                               x["lower_bound"], x["scale"], xd["initial_state"], xd["cu_seqlens"],
                               final_state=fin, batch=x["batch"])
    assert kda.kda_check_device_error() == 0
    return out, fin


def _oracle(x):
    return oracle.gdn_recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"],
                                x["lower_bound"], x["scale"], x["initial_state"], x["cu_seqlens"])


SMALL = [
    ("tiny_fixed_t256_h2", W.WORKLOADS[0]),
    ("one_chunk", W.custom([64], H=1, packed=False, init="normal")),
    ("partial_chunk", W.custom([37], H=2, packed=False, init="normal")),
    ("varlen_ragged", W.custom([70, 0, 129, 64, 1, 200, 17], H=3, init="normal")),
    ("many_heads", W.custom([300], H=20, packed=False, init=None)),
    ("steep_lb", W.custom([190], H=2, packed=False, init="normal", lower_bound=-20.0)),
    ("mild_lb", W.custom([190], H=2, packed=False, init="normal", lower_bound=-0.5)),
]


@pytest.mark.parametrize("name,w", SMALL, ids=[s[0] for s in SMALL])
def test_gdn_matches_oracle(name, w):
    kda = _kda()
    x = W.gdn_inputs(W.make_inputs(w))
    out, fin = _run(kda, x)
    ref_o, ref_f = _oracle(x)
    check(out, fin, ref_o, ref_f, name)


def test_gdn_unbounded_gate():
    kda = _kda()
    x = W.gdn_inputs(W.make_inputs(W.custom([150, 90], H=2, init="normal")))
    x["lower_bound"] = float("-inf")
    out, fin = _run(kda, x)
    ref_o, ref_f = _oracle(x)
    check(out, fin, ref_o, ref_f, "lb=-inf")


def test_gdn_split_and_resume():
    kda = _kda()
    w = W.custom([333], H=3, packed=False, init="normal")
    x = W.gdn_inputs(W.make_inputs(w))
    ref_o, ref_f = _oracle(x)
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


@pytest.mark.parametrize("wid", [2, 3])
def test_gdn_full_size_workloads(wid):
    """T=8192 H=96 varlen (no states) and 8 x 1024 H=64 with states, in full."""
    kda = _kda()
    w = W.WORKLOADS[wid]
    x = W.gdn_inputs(W.make_inputs(w))
    out, fin = _run(kda, x, want_final=True)
    ref_o, ref_f = _oracle(x)
    check(out, fin, ref_o, ref_f, "gdn " + w.name)
