"""Context-parallel prefill (gated_delta_rule_135_b200.cp) on two CPU ranks (gloo), with the
fp64 oracle standing in for the forward and a float64 matmul for the fold: the affine
decomposition S_out = A S_in + B over segments must reproduce the unsplit run."""
import os
import socket
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_fwd(gdn):
    import oracle

    def fwd(q, k, v, g, beta, A_log, dt_bias, lb, scale, init, cu, final_state=None, batch=1):
        f = oracle.gdn_recurrent if gdn else oracle.recurrent
        o, fin = f(q, k, v, g, beta, A_log, dt_bias, lb, scale,
                   None if init is None else init.double().numpy(), None)
        if final_state is not None:
            final_state.copy_(torch.from_numpy(fin))
        return torch.from_numpy(o), final_state
    return fwd


def _affine(A, S, B):
    return (A.double() @ S.double().reshape(A.shape) + B.double()).float()


def _load_cp():
    # the module is plain host code; load it without importing the CUDA binding
    import importlib.util
    spec = importlib.util.spec_from_file_location("kda_cp", os.path.join(ROOT, "gated_delta_rule_135_b200", "cp.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _rank_main(rank, world, port, gdn, cut, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import kda_workloads as W
    cp = _load_cp()
    x = W.make_inputs(W.custom([cut[-1]], H=2, packed=False, init="normal", wid=71))
    if gdn:
        x = W.gdn_inputs(x)
    lo, hi = cut[rank], cut[rank + 1]
    seg = {key: x[key][lo:hi].contiguous() for key in ("q", "k", "v", "g", "beta")}
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out, fin = cp.cp_prefill(seg["q"], seg["k"], seg["v"], seg["g"], seg["beta"], x["A_log"], x["dt_bias"],
                                 x["lower_bound"], x["scale"], x["initial_state"], gdn=gdn,
                                 fwd=_oracle_fwd(gdn), affine=_affine)
        results[rank] = (out.numpy(), fin.numpy())
    finally:
        dist.destroy_process_group()


def _check(gdn):
    import kda_workloads as W
    import oracle
    cut = [0, 170, 300]
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        results = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, gdn, cut, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=300)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(results)
    x = W.make_inputs(W.custom([cut[-1]], H=2, packed=False, init="normal", wid=71))
    if gdn:
        x = W.gdn_inputs(x)
    f = oracle.gdn_recurrent if gdn else oracle.recurrent
    ref_o, ref_f = f(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"], x["lower_bound"],
                     x["scale"], x["initial_state"], None)
    out = np.concatenate([res[0][0], res[1][0]])
    # the fold passes through fp32 maps, so agreement is at fp32 level
    assert oracle.rel_l2(out, ref_o) < 1e-6
    assert oracle.rel_l2(res[1][1], ref_f) < 1e-6


def test_cp_two_ranks_equals_unsplit_run():
    _check(gdn=False)


def test_cp_two_ranks_scalar_gate():
    _check(gdn=True)


def test_segment_offsets_are_chunk_aligned_and_cover():
    import kda_build
    kda_build.build()
    from gated_delta_rule_135_b200.cp import segment_offsets
    for T, R in ((700, 3), (131072, 8), (131072, 37), (64, 5), (1, 4), (1000, 1)):
        cuts = segment_offsets(T, R)
        assert cuts[0] == 0 and cuts[-1] == T
        assert all(b > a for a, b in zip(cuts, cuts[1:]))
        assert all(c % 64 == 0 for c in cuts[:-1])
        assert len(cuts) - 1 <= R


def test_choose_segments_fills_the_sms_only_when_heads_do_not():
    import kda_build
    kda_build.build()
    from gated_delta_rule_135_b200.cp import choose_segments
    # many (sequence, head) units already fill 148 SMs: no split
    assert choose_segments(8192, 96, 148) == 1
    assert choose_segments(1024, 64, 148) == 1
    # one long sequence with 32 heads: a split that fills the SMs
    R = choose_segments(131072, 32, 148)
    assert R >= 4 and R * 32 >= 128
