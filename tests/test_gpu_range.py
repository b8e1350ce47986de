"""GPU parity of kda_fwd outside the unit-norm regime of the standard workloads.

The fused kernel feeds fp16 tensor-core operands.  Those built from the state (S, Y, U, and
O through them) are kept in range by a power-of-two scale per value column of the state.  Each
column of S evolves on its own and the recurrence is linear in it, so this scaling is exact.
The operands built from one chunk's q and k need |q|, |k|, |beta k| and |q_r . k_i| below 2^15;
outside that range kda_fwd records KDA_DEVERR_RANGE and saturates instead of returning inf.

Tolerances are the parity tests' own: out rel-L2 2e-3 and final state rel-L2 1e-3, both
scale-free.  The max-abs bound 1e-2 is read scale-invariantly as max |out - ref| <= 1e-2
max(1, max |ref|): scaling V and the initial state by c scales every output by c, and a bf16
output of size 1e3 alone carries a rounding error of about 2.  At unit scale it is the plain
1e-2.
"""
import numpy as np
import pytest
import torch

import kda_workloads as W
import oracle
from kda_testutil import OUT_REL_L2, STATE_REL_L2, alloc_final, run_oracle, to_device

pytestmark = pytest.mark.gpu

KDA_DEVERR_RANGE = 0x8
OUT_SCALED_ABS = 1e-2


def _scaled_abs(o, ref):
    """max |o - ref| / max(1, max |ref|)."""
    return float(np.max(np.abs(o - ref)) / max(1.0, float(np.max(np.abs(ref)))))


def _kda():
    import kda_build as build
    build.build()
    import gated_delta_rule_135_b200 as kda
    return kda


def _check(out, fin, ref_out, ref_fin, label):
    o = out.float().cpu().numpy().astype(np.float64)
    f = fin.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(f)), f"{label}: non-finite result"
    e_rel = oracle.rel_l2(o, ref_out)
    e_abs = _scaled_abs(o, ref_out)
    e_st = oracle.rel_l2(f, ref_fin)
    msg = f"{label}: out rel-L2 {e_rel:.3e} scaled max-abs {e_abs:.3e} state rel-L2 {e_st:.3e}"
    assert e_rel <= OUT_REL_L2, msg
    assert e_abs <= OUT_SCALED_ABS, msg
    assert e_st <= STATE_REL_L2, msg


def _run(kda, x):
    xd = to_device(x)
    fin = alloc_final(xd, True)
    out, fin = kda.kda_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"],
                           x["lower_bound"], x["scale"], xd["initial_state"], xd["cu_seqlens"],
                           final_state=fin, batch=x["batch"])
    return out, fin


def _big_state(x, seed):
    """initial state ~ N(0, 1e3) with a few entries near 2e5 (above the fp16 maximum)."""
    gen = torch.Generator("cpu").manual_seed(seed)
    s = torch.randn(x["initial_state"].shape, generator=gen) * 1e3
    flat = s.view(-1)
    idx = torch.randint(0, flat.numel(), (64,), generator=gen)
    flat[idx] = torch.sign(torch.randn(64, generator=gen)) * 2e5
    return s


def _unnormalised(x, seed):
    """q, k ~ N(0, 1) per element (not L2-normalised); beta rescaled so that beta |k|^2 < 2
    (the condition under which each step (I - beta k k^T) is a contraction)."""
    gen = torch.Generator("cpu").manual_seed(seed)
    T, H, K = x["q"].shape
    y = dict(x)
    y["q"] = torch.randn(T, H, K, generator=gen).to(torch.bfloat16)
    k = torch.randn(T, H, K, generator=gen).to(torch.bfloat16)
    y["k"] = k
    kn2 = k.float().pow(2).sum(-1)
    y["beta"] = (x["beta"] * 1.9 / kn2).contiguous()
    return y


CASES = ["big_state", "v_times_1e3", "unnormalised_qk", "all_three", "all_three_lb_5_3"]


@pytest.mark.parametrize("case", CASES)
def test_range_matches_oracle(case):
    kda = _kda()
    lb = -5.3 if case.endswith("lb_5_3") else -5.0
    w = W.custom([300, 77, 130], H=3, init="normal", lower_bound=lb, wid=41)
    x = W.make_inputs(w)
    if case in ("big_state", "all_three", "all_three_lb_5_3"):
        x["initial_state"] = _big_state(x, 7)
    if case in ("v_times_1e3", "all_three", "all_three_lb_5_3"):
        x["v"] = (x["v"].float() * 1e3).to(torch.bfloat16)
    if case in ("unnormalised_qk", "all_three", "all_three_lb_5_3"):
        x = _unnormalised(x, 9)
    out, fin = _run(kda, x)
    bits = kda.kda_check_device_error()
    assert bits == 0, f"device error bits {bits:#x}"
    ref_o, ref_f = run_oracle(x)
    _check(out, fin, ref_o, ref_f, case)


def test_range_state_grows_then_decays():
    """A state driven far above the fp16 range by large values (|S| ~ 1e5), then decayed by a
    gate held at the lower bound: the per-column scale moves up and back down.  Each segment
    is checked against its own scale (the late outputs are about 1e-3 in size, so a scale left
    high would lose them to fp16 subnormals)."""
    kda = _kda()
    w = W.custom([640], H=2, packed=False, init="normal", wid=43)
    x = W.make_inputs(w)
    v = x["v"].float()
    v[:192] *= 2e5          # large values early ...
    x["v"] = v.to(torch.bfloat16)
    g = x["g"].clone()
    g[192:] += 4.0          # ... then a gate at the lower bound, so the state shrinks
    x["g"] = g
    out, fin = _run(kda, x)
    assert kda.kda_check_device_error() == 0
    ref_o, ref_f = run_oracle(x)
    o = out.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(o))
    for a, b in ((0, 192), (256, 640)):
        seg, ref = o[a:b], ref_o[a:b]
        e_rel = oracle.rel_l2(seg, ref)
        e_abs = _scaled_abs(seg, ref)
        assert e_rel <= OUT_REL_L2 and e_abs <= OUT_SCALED_ABS, \
            f"tokens {a}-{b}: rel-L2 {e_rel:.3e} scaled max-abs {e_abs:.3e}"
    e_st = oracle.rel_l2(fin.cpu().numpy().astype(np.float64), ref_f)
    assert e_st <= STATE_REL_L2, f"state rel-L2 {e_st:.3e}"


def test_steep_gate_with_large_keys():
    """The steepest clamp the fused kernel takes (-9.5) with entries of q and k up to ~50 (|q . k|
    still below 2^15) and most gates at the clamp: every decayed operand stays finite (factors are
    taken around the middle of each 16-token block), and the result matches the oracle."""
    kda = _kda()
    w = W.custom([300, 90], H=2, init="normal", lower_bound=-9.5, wid=49)
    x = _unnormalised(W.make_inputs(w), 13)
    x["k"] = (x["k"].float() * 10.0).to(torch.bfloat16)
    x["q"] = (x["q"].float() * 10.0).to(torch.bfloat16)
    kn2 = x["k"].float().pow(2).sum(-1)
    x["beta"] = (torch.rand(kn2.shape, generator=torch.Generator("cpu").manual_seed(17)) * 1.9 / kn2).contiguous()
    x["g"] = x["g"] + 3.0       # softplus(g + dt_bias) large: log a at the clamp for most tokens
    out, fin = _run(kda, x)
    assert kda.kda_check_device_error() == 0
    ref_o, ref_f = run_oracle(x)
    _check(out, fin, ref_o, ref_f, "steep gate, large keys")


def test_out_of_range_keys_are_flagged_not_inf():
    """Keys far outside the operating range (|k| ~ 1e5): the kernel saturates instead of
    producing inf or NaN, and reports KDA_DEVERR_RANGE."""
    kda = _kda()
    w = W.custom([200], H=2, packed=False, init="normal", wid=45)
    x = W.make_inputs(w)
    x["k"] = (x["k"].float() * 1e6).to(torch.bfloat16)
    x["beta"] = x["beta"] * 1e-12
    out, fin = _run(kda, x)
    bits = kda.kda_check_device_error()
    assert bits & KDA_DEVERR_RANGE, f"expected the range bit, got bits {bits:#x}"
    assert torch.isfinite(out.float()).all() and torch.isfinite(fin).all()


@pytest.mark.parametrize("lb", [-5.0, -20.0])
def test_range_scalar_gate_matches_oracle(lb):
    """kda_gdn_fwd (one decay per token-head) shares the state chain and its per-column scale:
    huge initial states and v x 1e3 against the fp64 scalar-gate oracle."""
    kda = _kda()
    w = W.custom([300, 77, 130], H=3, init="normal", lower_bound=lb, wid=47)
    x = W.gdn_inputs(W.make_inputs(w))
    x["initial_state"] = _big_state(x, 11)
    x["v"] = (x["v"].float() * 1e3).to(torch.bfloat16)
    xd = to_device(x)
    fin = alloc_final(xd, True)
    out, fin = kda.kda_gdn_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"],
                               x["lower_bound"], x["scale"], xd["initial_state"], xd["cu_seqlens"],
                               final_state=fin, batch=x["batch"])
    bits = kda.kda_check_device_error()
    assert bits == 0, f"device error bits {bits:#x}"
    ref_o, ref_f = oracle.gdn_recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"],
                                        x["lower_bound"], x["scale"], x["initial_state"], x["cu_seqlens"])
    _check(out, fin, ref_o, ref_f, f"scalar gate lb={lb}")
