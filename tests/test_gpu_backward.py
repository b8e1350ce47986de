"""GPU parity of the backward kda_bwd against the fp64 backward oracle.

The oracle's gradients are pinned by central finite differences (test_oracle_backward).
Tolerance: every gradient rel-L2 <= 1e-3 against fp64.  Both sides read the same bf16
q, k, v, d_out and fp32 g, beta, gate parameters, states and d_final_state; the
library computes in fp32, so its error is rounding accumulated over the chunk algebra
(tens of fp32 operations on O(1) values, amplified by T = (I + A)^-1 whose entries stay
O(1) for beta in (0, 1) and unit-norm keys): ~1e-5 typical, 1e-3 leaves a wide margin
while a dropped term or a wrong sign gives O(1)."""
import numpy as np
import pytest
import torch

import kda_workloads as W
import oracle
from oracle import backward as OB
from kda_testutil import to_device

pytestmark = pytest.mark.gpu

GRAD_REL_L2 = 1e-3
NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dA_log", "ddt_bias", "d_initial_state")


def _kda():
    import kda_build as build
    build.build()
    import gated_delta_rule_135_b200 as kda
    return kda


def _gpu(kda, x, dO, dF, want_d_initial=True, **kw):
    xd = to_device(x)
    gr = kda.kda_bwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"],
                     x["lower_bound"], x["scale"], dO.cuda(), xd["initial_state"], xd["cu_seqlens"],
                     None if dF is None else dF.cuda(), want_d_initial=want_d_initial, batch=x["batch"], **kw)
    assert kda.kda_check_device_error() == 0
    return {n: t.cpu() for n, t in gr.items()}


def _oracle(x, dO, dF, chunked=False):
    f = OB.grads_chunked if chunked else OB.grads_autograd
    cu = x["cu_seqlens"]
    if cu is None:   # the fixed layout: batch sequences of seqlen tokens each
        cu = torch.arange(x["batch"] + 1, dtype=torch.int32) * x["seqlen"]
    r = f(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"], x["lower_bound"], x["scale"],
          x["initial_state"], cu, dO, dF)
    return dict(zip(NAMES, r))


def _compare(got, ref, label, names=NAMES):
    errs = {}
    for n in names:
        if n not in got or got[n] is None:
            continue
        a = got[n].numpy().astype(np.float64).reshape(ref[n].shape)
        assert np.all(np.isfinite(a)), f"{label} {n}: non-finite"
        errs[n] = oracle.rel_l2(a, ref[n])
    bad = {n: e for n, e in errs.items() if not e <= GRAD_REL_L2}
    assert not bad, f"{label}: rel-L2 above {GRAD_REL_L2}: {bad} (all: {errs})"
    return errs


SMALL = [
    ("one_chunk", dict(seq_lens=[64], H=1, packed=False, init="normal")),
    ("partial_chunk", dict(seq_lens=[37], H=2, packed=False, init="normal")),
    ("varlen_ragged", dict(seq_lens=[70, 0, 129, 64, 1, 200, 17], H=2, init="normal")),
    ("fixed_batch", dict(seq_lens=[150, 150], H=2, packed=False, init=None)),
    ("lb_mild", dict(seq_lens=[190], H=2, packed=False, init="normal", lower_bound=-1.0)),
    ("lb_steep", dict(seq_lens=[130, 66], H=2, init="normal", lower_bound=-20.0)),
    ("lb_none", dict(seq_lens=[100], H=1, packed=False, init="normal", lower_bound=float("-inf"))),
]


@pytest.mark.parametrize("name,kw", SMALL, ids=[s[0] for s in SMALL])
def test_backward_matches_autograd_oracle(name, kw):
    kda = _kda()
    w = W.custom(wid=300 + len(name), **kw)
    x = W.make_inputs(w)
    dO, dF = W.cotangents(w)
    got = _gpu(kda, x, dO, dF)
    _compare(got, _oracle(x, dO, dF), name)


def test_backward_without_state_gradients():
    """No d_final_state (zero) and no d_initial_state requested."""
    kda = _kda()
    w = W.custom([140, 60], H=2, init=None, wid=321)
    x = W.make_inputs(w)
    dO, _ = W.cotangents(w)
    got = _gpu(kda, x, dO, None, want_d_initial=False)
    assert "d_initial_state" not in got
    _compare(got, _oracle(x, dO, None), "no-state-grads")


def test_backward_in_place_state_gradient():
    kda = _kda()
    w = W.custom([90, 40], H=2, init="normal", wid=322)
    x = W.make_inputs(w)
    dO, dF = W.cotangents(w)
    ref = _oracle(x, dO, dF)
    xd = to_device(x)
    st = dF.cuda().clone()
    kda.kda_bwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"], x["lower_bound"],
                x["scale"], dO.cuda(), xd["initial_state"], xd["cu_seqlens"], st, grads={"d_initial_state": st})
    assert oracle.rel_l2(st.cpu().numpy().astype(np.float64), ref["d_initial_state"]) <= GRAD_REL_L2


def test_backward_is_deterministic():
    kda = _kda()
    w = W.custom([300, 200], H=3, init="normal", wid=323)
    x = W.make_inputs(w)
    dO, dF = W.cotangents(w)
    a = _gpu(kda, x, dO, dF)
    b = _gpu(kda, x, dO, dF)
    for n in NAMES:
        assert torch.equal(a[n], b[n]), n


def test_backward_empty_sequences_only():
    """Ttot = 0: parameter gradients are zero and d_initial_state = d_final_state."""
    kda = _kda()
    w = W.custom([0, 0], H=2, init="normal", wid=324)
    x = W.make_inputs(w)
    dO, dF = W.cotangents(w)
    got = _gpu(kda, x, dO, dF)
    assert torch.count_nonzero(got["dA_log"]) == 0 and torch.count_nonzero(got["ddt_bias"]) == 0
    assert torch.equal(got["d_initial_state"], dF)


@pytest.mark.parametrize("wid", [2, 3, 4])
def test_backward_full_size_sampled_heads(wid):
    """The full workload on the GPU; heads 0, H/2 and H-1 (one head, 17, for the 131072-token
    sequence) against the chunked fp64 oracle (pinned to autograd), which treats every head
    independently."""
    kda = _kda()
    w = W.WORKLOADS[wid]
    x = W.make_inputs(w)
    dO, dF = W.cotangents(w)
    if not w.final:
        dF = None
    got = _gpu(kda, x, dO, dF)
    heads = [17] if w.T > 100000 else [0, w.H // 2, w.H - 1]
    xs = dict(x)
    for key in ("q", "k", "v", "g", "beta"):
        xs[key] = x[key][:, heads].contiguous()
    xs["A_log"], xs["dt_bias"] = x["A_log"][heads], x["dt_bias"][heads]
    if x["initial_state"] is not None:
        xs["initial_state"] = x["initial_state"][:, heads].contiguous()
    ref = _oracle(xs, dO[:, heads].contiguous(), None if dF is None else dF[:, heads].contiguous(), chunked=True)
    sub = {}
    for n in NAMES:
        t = got[n]
        if n in ("dA_log", "ddt_bias"):
            sub[n] = t[heads]
        elif n == "d_initial_state":
            sub[n] = t[:, heads]
        else:
            sub[n] = t[:, heads]
    _compare(sub, ref, w.name)


