"""GPU parity of kda_decode (one recurrent step per sequence, in place on the
state) against the fp64 oracle's token-by-token recurrence."""
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


def _step_inputs(xd, B, T, t):
    """Token t of each of the B fixed-length sequences: [B, H, ...] views."""
    rows = torch.arange(B, device=xd["q"].device) * T + t
    return {key: xd[key][rows].contiguous() for key in ("q", "k", "v", "g", "beta")}


@pytest.mark.parametrize("B,T,H", [(4, 5, 3), (2, 70, 2)])
def test_decode_steps_match_recurrence(B, T, H):
    kda = _kda()
    w = W.custom([T] * B, H=H, packed=False, init="normal", wid=51)
    x = W.make_inputs(w)
    xd = to_device(x)
    ref_o, ref_f = oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"],
                                    x["lower_bound"], x["scale"], x["initial_state"],
                                    oracle.fixed_offsets(B, T))
    state = xd["initial_state"].clone()
    outs = []
    for t in range(T):
        s = _step_inputs(xd, B, T, t)
        outs.append(kda.kda_decode(s["q"], s["k"], s["v"], s["g"], s["beta"], xd["A_log"], xd["dt_bias"],
                                   x["lower_bound"], x["scale"], state))
    torch.cuda.synchronize()
    o = torch.stack(outs, dim=1).reshape(B * T, H, 128).float().cpu().numpy().astype(np.float64)
    assert oracle.rel_l2(o, ref_o) <= OUT_REL_L2
    assert oracle.max_abs(o, ref_o) <= OUT_MAX_ABS
    assert oracle.rel_l2(state.cpu().numpy(), ref_f) <= STATE_REL_L2


def test_prefill_then_decode_equals_longer_prefill():
    kda = _kda()
    B, T, H = 3, 200, 4
    w = W.custom([T + 1] * B, H=H, packed=False, init="normal", wid=52)
    x = W.make_inputs(w)
    ref_o, ref_f = oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"],
                                    x["lower_bound"], x["scale"], x["initial_state"],
                                    oracle.fixed_offsets(B, T + 1))
    xd = to_device(x)
    # prefill of the first T tokens of every sequence with the fused kernel
    idx = torch.cat([torch.arange(b * (T + 1), b * (T + 1) + T) for b in range(B)]).cuda()
    pre = {key: xd[key][idx].contiguous() for key in ("q", "k", "v", "g", "beta")}
    state = torch.empty_like(xd["initial_state"])
    kda.kda_fwd(pre["q"], pre["k"], pre["v"], pre["g"], pre["beta"], xd["A_log"], xd["dt_bias"],
                x["lower_bound"], x["scale"], xd["initial_state"], None, final_state=state, batch=B)
    s = _step_inputs(xd, B, T + 1, T)
    o = kda.kda_decode(s["q"], s["k"], s["v"], s["g"], s["beta"], xd["A_log"], xd["dt_bias"],
                       x["lower_bound"], x["scale"], state)
    torch.cuda.synchronize()
    ref_last = ref_o.reshape(B, T + 1, H, 128)[:, T]
    o = o.float().cpu().numpy().astype(np.float64)
    assert oracle.rel_l2(o, ref_last) <= OUT_REL_L2
    assert oracle.rel_l2(state.cpu().numpy(), ref_f) <= STATE_REL_L2


@pytest.mark.parametrize("B,T,H", [(3, 6, 4)])
def test_gdn_decode_steps_match_recurrence(B, T, H):
    kda = _kda()
    w = W.custom([T] * B, H=H, packed=False, init="normal", wid=53)
    x = W.gdn_inputs(W.make_inputs(w))
    xd = to_device(x)
    ref_o, ref_f = oracle.gdn_recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"],
                                        x["dt_bias"], x["lower_bound"], x["scale"], x["initial_state"],
                                        oracle.fixed_offsets(B, T))
    state = xd["initial_state"].clone()
    outs = []
    for t in range(T):
        s = _step_inputs(xd, B, T, t)
        outs.append(kda.kda_gdn_decode(s["q"], s["k"], s["v"], s["g"], s["beta"], xd["A_log"], xd["dt_bias"],
                                       x["lower_bound"], x["scale"], state))
    torch.cuda.synchronize()
    o = torch.stack(outs, dim=1).reshape(B * T, H, 128).float().cpu().numpy().astype(np.float64)
    assert oracle.rel_l2(o, ref_o) <= OUT_REL_L2
    assert oracle.max_abs(o, ref_o) <= OUT_MAX_ABS
    assert oracle.rel_l2(state.cpu().numpy(), ref_f) <= STATE_REL_L2
