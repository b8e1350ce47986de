"""Context-parallel prefill emulated on one GPU: three segments of one sequence, each
taken through the library's steps (segment maps from two forwards, the fold with
kda_state_affine, the final forward) in turn, with no rank waiting on another.  The
concatenated outputs and the last segment's final state must match the fp64 oracle on the
unsplit sequence."""
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
    from gated_delta_rule_135_b200 import cp
    return kda, cp


@pytest.mark.parametrize("gdn", [False, True], ids=["kda", "scalar_gate"])
def test_cp_three_segments_emulated(gdn):
    kda, cp = _kda()
    cut = [0, 300, 517, 700]
    H = 3
    x = W.make_inputs(W.custom([cut[-1]], H=H, packed=False, init="normal", wid=72))
    if gdn:
        x = W.gdn_inputs(x)
    xd = to_device(x)
    fwd = kda.kda_gdn_fwd if gdn else kda.kda_fwd
    # slices at token offsets: beta is only 4-byte aligned there, which the library accepts;
    # q, k, v, g rows are 16-byte multiples
    segs = [{key: xd[key][lo:hi] for key in ("q", "k", "v", "g", "beta")}
            for lo, hi in zip(cut[:-1], cut[1:])]
    maps = torch.stack([cp.segment_maps(fwd, s["q"], s["k"], s["v"], s["g"], s["beta"], xd["A_log"],
                                        xd["dt_bias"], x["lower_bound"], x["scale"]) for s in segs])
    outs = []
    fin = None
    for r, s in enumerate(segs):
        S = cp.fold(kda.kda_state_affine, maps, xd["initial_state"], r, H, xd["q"].device)
        fin = torch.empty(1, H, 128, 128, device=xd["q"].device)
        o, fin = fwd(s["q"], s["k"], s["v"], s["g"], s["beta"], xd["A_log"], xd["dt_bias"], x["lower_bound"],
                     x["scale"], S, None, final_state=fin)
        outs.append(o)
    assert kda.kda_check_device_error() == 0
    f = oracle.gdn_recurrent if gdn else oracle.recurrent
    ref_o, ref_f = f(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"], x["lower_bound"],
                     x["scale"], x["initial_state"], None)
    o = torch.cat(outs).float().cpu().numpy().astype(np.float64)
    assert oracle.rel_l2(o, ref_o) <= OUT_REL_L2
    assert oracle.max_abs(o, ref_o) <= OUT_MAX_ABS
    assert oracle.rel_l2(fin.cpu().numpy(), ref_f) <= STATE_REL_L2


def test_state_affine_matches_matmul():
    kda, _ = _kda()
    g = torch.Generator("cpu").manual_seed(5)
    A, S, B = (torch.randn(4, 128, 128, generator=g) for _ in range(3))
    out = kda.kda_state_affine(A.cuda(), S.cuda(), B.cuda())
    ref = (A.double() @ S.double() + B.double())
    assert torch.allclose(out.cpu().double(), ref, rtol=1e-5, atol=1e-4)


@pytest.mark.parametrize("gdn", [False, True], ids=["kda", "scalar_gate"])
def test_segmented_prefill_matches_oracle(gdn):
    """One sequence split into segments run as one varlen batch per pass (maps, fold, final)."""
    kda, cp = _kda()
    H = 3
    x = W.make_inputs(W.custom([700], H=H, packed=False, init="normal", wid=73))
    if gdn:
        x = W.gdn_inputs(x)
    xd = to_device(x)
    assert cp.segment_offsets(700, 3) == [0, 256, 512, 700]
    ws = {}
    for _ in range(2):          # the second call reuses the cached buffers
        out, fin = cp.segmented_prefill(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"],
                                        xd["dt_bias"], x["lower_bound"], x["scale"], xd["initial_state"],
                                        segments=3, gdn=gdn, workspace=ws)
    assert kda.kda_check_device_error() == 0
    f = oracle.gdn_recurrent if gdn else oracle.recurrent
    ref_o, ref_f = f(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"], x["lower_bound"],
                     x["scale"], x["initial_state"], None)
    o = out.float().cpu().numpy().astype(np.float64)
    assert oracle.rel_l2(o, ref_o) <= OUT_REL_L2
    assert oracle.max_abs(o, ref_o) <= OUT_MAX_ABS
    assert oracle.rel_l2(fin.cpu().numpy(), ref_f) <= STATE_REL_L2


def test_segmented_prefill_long_sequence_full_size():
    """T = 131072, H = 32 with states, split in 8 segments, against the fp64 oracle."""
    kda, cp = _kda()
    w = W.WORKLOADS[4]
    x = W.make_inputs(w)
    xd = to_device(x)
    out, fin = cp.segmented_prefill(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"],
                                    x["lower_bound"], x["scale"], xd["initial_state"], segments=8)
    assert kda.kda_check_device_error() == 0
    ref_o, ref_f = oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"],
                                    x["lower_bound"], x["scale"], x["initial_state"], None)
    o = out.float().cpu().numpy().astype(np.float64)
    assert oracle.rel_l2(o, ref_o) <= OUT_REL_L2
    assert oracle.max_abs(o, ref_o) <= OUT_MAX_ABS
    assert oracle.rel_l2(fin.cpu().numpy(), ref_f) <= STATE_REL_L2


@pytest.mark.parametrize("gdn", [False, True], ids=["kda", "scalar_gate"])
def test_library_splits_one_long_sequence(gdn):
    """kda_fwd / kda_gdn_fwd on one 16384-token sequence with two heads (2 of 148 SMs busy
    unsplit) take the segmented decomposition inside the library; the output and the final state
    (written over the initial state, in place) match the fp64 oracle on the unsplit sequence."""
    kda, _ = _kda()
    H, T = 2, 16384
    R = kda.kda_fwd_segments(H, T)
    assert R > 1, "the library should split this call"
    assert kda.kda_fwd_segments(H, T, varlen=True) == 1 and kda.kda_fwd_segments(H, T // 2, batch=2) == 1
    x = W.make_inputs(W.custom([T], H=H, packed=False, init="normal", wid=77))
    if gdn:
        x = W.gdn_inputs(x)
    xd = to_device(x)
    fin = xd["initial_state"].clone()
    fwd = kda.kda_gdn_fwd if gdn else kda.kda_fwd
    out, fin = fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"], x["lower_bound"],
                   x["scale"], fin, None, final_state=fin, batch=1)
    assert kda.kda_check_device_error() == 0
    f = oracle.gdn_recurrent if gdn else oracle.recurrent
    ref_o, ref_f = f(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"], x["lower_bound"],
                     x["scale"], x["initial_state"], None)
    o = out.float().cpu().numpy().astype(np.float64)
    assert oracle.rel_l2(o, ref_o) <= OUT_REL_L2, f"R={R}"
    assert oracle.max_abs(o, ref_o) <= OUT_MAX_ABS, f"R={R}"
    assert oracle.rel_l2(fin.cpu().numpy(), ref_f) <= STATE_REL_L2, f"R={R}"
