"""Shared helpers of the GPU parity tests: move seeded inputs to the device,
call the library, run the oracle on the same inputs, and apply the tolerances.

Tolerances (against the fp64 oracle, out compared after the library's bf16
rounding):  out rel-L2 <= 2e-3 and max-abs <= 1e-2; final state rel-L2 <= 1e-3.
"""
import numpy as np
import torch

import oracle

OUT_REL_L2 = 2e-3
OUT_MAX_ABS = 1e-2
STATE_REL_L2 = 1e-3


def to_device(x: dict, device="cuda") -> dict:
    d = dict(x)
    for key in ("q", "k", "v", "g", "beta", "A_log", "dt_bias", "initial_state", "cu_seqlens"):
        if d.get(key) is not None:
            d[key] = d[key].to(device).contiguous()
    return d


def run_oracle(x: dict, nthreads: int = 0):
    return oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"],
                            x["lower_bound"], x["scale"], x["initial_state"], x["cu_seqlens"],
                            nthreads=nthreads)


def alloc_final(xd: dict, want: bool):
    if not want:
        return None
    H = xd["q"].shape[-2]
    return torch.full((xd["N"], H, 128, 128), float("nan"), device=xd["q"].device)


def check(out, fin, ref_out, ref_fin, label=""):
    o = out.float().cpu().numpy().astype(np.float64)
    e_rel = oracle.rel_l2(o, ref_out)
    e_abs = oracle.max_abs(o, ref_out)
    msg = f"{label}: out rel-L2 {e_rel:.3e} max-abs {e_abs:.3e}"
    assert np.all(np.isfinite(o)), msg + " (non-finite output)"
    assert e_rel <= OUT_REL_L2, msg
    assert e_abs <= OUT_MAX_ABS, msg
    e_st = None
    if fin is not None:
        f = fin.cpu().numpy().astype(np.float64)
        e_st = oracle.rel_l2(f, ref_fin)
        assert np.all(np.isfinite(f)), msg + " (non-finite state)"
        assert e_st <= STATE_REL_L2, msg + f" state rel-L2 {e_st:.3e}"
    return e_rel, e_abs, e_st


BWD_NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dA_log", "ddt_bias", "d_initial_state")


def head_slice(x: dict, dO, dF, heads):
    """The inputs and cotangents of the given heads only (the recurrence treats heads independently)."""
    xs = dict(x)
    for key in ("q", "k", "v", "g", "beta"):
        xs[key] = x[key][:, heads].contiguous()
    xs["A_log"], xs["dt_bias"] = x["A_log"][heads].contiguous(), x["dt_bias"][heads].contiguous()
    if x["initial_state"] is not None:
        xs["initial_state"] = x["initial_state"][:, heads].contiguous()
    return xs, dO[:, heads].contiguous(), None if dF is None else dF[:, heads].contiguous()


def backward_oracle(args):
    """Chunked fp64 backward oracle on one set of heads (one task of a spawn pool)."""
    from oracle import backward as OB
    x, dO, dF = args
    torch.set_num_threads(1)
    cu = x["cu_seqlens"]
    if cu is None:   # the fixed layout: batch sequences of seqlen tokens each
        cu = torch.arange(x["batch"] + 1, dtype=torch.int32) * x["seqlen"]
    r = OB.grads_chunked(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"], x["lower_bound"],
                         x["scale"], x["initial_state"], cu, dO, dF)
    return dict(zip(BWD_NAMES, r))


def backward_oracle_all_heads(x: dict, dO, dF, H: int, procs: int = 0):
    """The backward oracle for every head, one head per task on a spawn pool (spawn: the parent
    has a CUDA context, which a forked child must not inherit).  Each worker runs single-threaded
    (its BLAS and OpenMP pools too): one process per core, not one thread pool per process."""
    import multiprocessing as mp
    import os
    procs = procs or min(H, len(os.sched_getaffinity(0)))
    tasks = [head_slice(x, dO, dF, [h]) for h in range(H)]
    # read by the children at start-up: one thread each, and glibc malloc keeps the oracle's
    # many short-lived arrays on its heap instead of mapping and unmapping pages for each
    env = {"OMP_NUM_THREADS": "1", "OPENBLAS_NUM_THREADS": "1", "MKL_NUM_THREADS": "1",
           "MALLOC_MMAP_THRESHOLD_": str(1 << 30), "MALLOC_TRIM_THRESHOLD_": str(1 << 32)}
    saved = {k: os.environ.get(k) for k in env}
    os.environ.update(env)
    try:
        with mp.get_context("spawn").Pool(procs) as pool:
            return pool.map(backward_oracle, tasks, chunksize=1)
    finally:
        for k, v in saved.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
