"""GPU parity of the staged path (kda_fwd_staged): each stage against the fp64
chunked oracle's intermediates, and the whole forward against the fp64
recurrent oracle."""
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


CASES = [
    ("tiny_fixed", W.WORKLOADS[0]),
    ("varlen_ragged", W.custom([70, 0, 129, 64, 1, 200], H=3, init="normal")),
    ("steep_gate_lb-20", W.custom([150, 90], H=2, init="normal", lower_bound=-20.0)),
    ("unclamped_lb-inf", W.custom([130], H=2, packed=False, init=None,
                                  lower_bound=-float("inf"))),
]


@pytest.mark.parametrize("name,w", CASES, ids=[c[0] for c in CASES])
def test_staged_end_to_end(name, w):
    kda = _kda()
    x = W.make_inputs(w)
    xd = to_device(x)
    fin = alloc_final(xd, True)
    out, fin, _ = kda.kda_fwd_staged(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"],
                                     xd["dt_bias"], x["lower_bound"], x["scale"],
                                     xd["initial_state"], xd["cu_seqlens"], final_state=fin,
                                     batch=x["batch"])
    assert kda.kda_check_device_error() == 0
    ref_o, ref_f = run_oracle(x)
    check(out, fin, ref_o, ref_f, name)


def test_staged_stages_match_chunked_oracle():
    kda = _kda()
    w = W.custom([70, 0, 129, 64], H=2, init="normal")
    x = W.make_inputs(w)
    xd = to_device(x)
    fin = alloc_final(xd, True)
    out, fin, ws = kda.kda_fwd_staged(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"],
                                      xd["dt_bias"], x["lower_bound"], x["scale"],
                                      xd["initial_state"], xd["cu_seqlens"], final_state=fin)
    torch.cuda.synchronize()
    T, H = w.T, w.H
    L = ws.layout
    gamma = ws.view("gamma", torch.float32, (T, H, 128)).cpu().double().numpy()
    wm = ws.view("w", torch.float32, (T, H, 128)).cpu().double().numpy()
    ut = ws.view("u_tilde", torch.float32, (T, H, 128)).cpu().double().numpy()
    pm = ws.view("p", torch.float32, (T, H, 64)).cpu().double().numpy()
    um = ws.view("u", torch.float32, (T, H, 128)).cpu().double().numpy()
    table = ws.view("chunk_table", torch.int32, (L.max_chunks * 4 + 1,)).cpu().numpy()
    count = int(table[-1])
    table = table[:-1].reshape(-1, 4)
    cs = ws.view("chunk_states", torch.float32, (L.max_chunks, H, 128, 128)).cpu().double().numpy()
    _, _, stages = oracle.chunked(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"],
                                  x["dt_bias"], x["lower_bound"], x["scale"], x["initial_state"],
                                  x["cu_seqlens"], keep_stages=True)
    # the chunk table lists every chunk once, in sequence order
    expect_tab = []
    cu = x["cu_seqlens"].tolist()
    for n in range(w.N):
        for j, t0 in enumerate(range(cu[n], cu[n + 1], 64)):
            expect_tab.append((n, t0, min(64, cu[n + 1] - t0), j))
    assert count == len(expect_tab)
    assert [tuple(r) for r in table[:count]] == expect_tab
    for ci, (n, t0, ln, j) in enumerate(expect_tab):
        for h in range(H):
            st = stages[(n, h)][j]
            sl = slice(t0, t0 + ln)
            np.testing.assert_allclose(gamma[sl, h], st["Gamma"], rtol=2e-6, atol=2e-5)
            assert oracle.rel_l2(wm[sl, h], st["W"]) < 2e-5
            assert oracle.rel_l2(ut[sl, h], st["Ut"]) < 2e-5
            p_ref = np.zeros((ln, 64))
            p_ref[:, :ln] = st["P"]
            assert oracle.rel_l2(pm[sl, h], p_ref) < 2e-5
            assert oracle.rel_l2(um[sl, h], st["U"]) < 1e-4
            assert oracle.rel_l2(cs[ci, h], st["S0"]) < 1e-4 or np.abs(st["S0"]).max() == 0


def test_staged_workspace_too_small_is_rejected():
    kda = _kda()
    x = W.make_inputs(W.WORKLOADS[0])
    xd = to_device(x)
    ws = kda.staged_workspace(xd["q"])
    ws.buffer = ws.buffer[:1024]
    with pytest.raises(kda.KdaError) as e:
        kda.kda_fwd_staged(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"],
                           xd["dt_bias"], x["lower_bound"], x["scale"], workspace=ws)
    assert e.value.status == 6
