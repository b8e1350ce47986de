"""Per-phase cycle counts of the fused prefill kernel (a profiling aid, not part of the ABI).

Builds the instrumented library (``build.py --phase-clocks``: the same kernel with clock64()
marks between its phases, accumulated per CTA), runs one workload through it and prints the
average cycles per 64-token chunk of each phase, for the aux warps (thread 128), the element
warps (thread 256) and the state chain (thread 0).  Run it by path from the repository root (importing the package loads the
product library, so this script sets KDA_LIBRARY before it imports the package):

    python gated_delta_rule_135_b200/phase_clocks.py [--workload 2] [--gdn]

The instrumented build is slower than the product build (the marks serialise a little); compare
phases with each other, not the printed kernel time with the bench.
"""
from __future__ import annotations

import argparse
import ctypes
import os
import sys

_HERE = os.path.dirname(os.path.abspath(__file__))
_ROOT = os.path.dirname(_HERE)

# index = slot of the kernel's phase marks; each counts the cycles since the previous mark
# of the same role
PHASES = [
    ("aux", "wait for A/P product, last [S|O], chunk data"),
    ("aux", "A / P read-out"),
    ("aux", "solve L0 (diagonal blocks)"),
    ("aux", "solve L1 + L2, T written"),
    ("-", "(unused)"),
    ("aux", "meet the other aux warps"),
    ("-", "(unused)"),
    ("-", "(unused)"),
    ("-", "(unused)"),
    ("chain", "wait for the previous [S|O] MMA"),
    ("chain", "output of the previous chunk"),
    ("chain", "wait for A/P operands and read-out, issue"),
    ("chain", "(between marks)"),
    ("chain", "wait for the chunk's operands, next TMA"),
    ("chain", "S^T -> fp16, [O|Y] MMA, S <- S Diag(gamma_C)"),
    ("chain", "wait [O|Y], Y^T += beta V^T -> fp16"),
    ("chain", "wait T, U MMA, wait U"),
    ("chain", "U -> fp16, [S|O] MMA issue"),
    ("elem", "beta, block products / gate scan"),
    ("elem", "wait for the inputs and the last A/P MMA"),
    ("elem", "A/P operand tiles, P diagonal"),
    ("elem", "wait for the last [S|O] MMA"),
    ("elem", "B1, Khat, V^T tiles, metadata"),
    ("elem", "next chunk: beta, gate"),
]


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--workload", type=int, default=2)
    ap.add_argument("--gdn", action="store_true", help="the scalar-gate forward (kda_gdn_fwd)")
    args = ap.parse_args(argv)

    sys.path.insert(0, _ROOT)
    import kda_build
    lib_path = kda_build.build(phase_clocks=True)
    os.environ["KDA_LIBRARY"] = lib_path
    import torch

    import gated_delta_rule_135_b200 as kda
    import kda_workloads as W

    w = W.WORKLOADS[args.workload]
    x = W.make_inputs(w)
    if args.gdn:
        x = W.gdn_inputs(x)
    xd = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    fin = torch.empty(w.N, w.H, 128, 128, device="cuda") if w.final else None
    fwd = kda.kda_gdn_fwd if args.gdn else kda.kda_fwd

    def step():
        fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"], x["lower_bound"],
            x["scale"], xd["initial_state"], xd["cu_seqlens"], final_state=fin, batch=x["batch"])

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    lib = kda.lib()
    lib.kda_debug_pipe_phase_cycles.restype = ctypes.c_int
    buf = (ctypes.c_ulonglong * len(PHASES))()
    if lib.kda_debug_pipe_phase_cycles(buf) != len(PHASES):   # clears the counters
        raise RuntimeError("phase counters not available in this build")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    step()
    e1.record()
    torch.cuda.synchronize()
    if lib.kda_debug_pipe_phase_cycles(buf) != len(PHASES):
        raise RuntimeError("reading the phase counters failed")
    chunks = sum((s + 63) // 64 for s in w.seq_lens) * w.H
    print(f"instrumented kernel {e0.elapsed_time(e1):.3f} ms, {chunks} chunk-heads")
    tot = {"aux": 0.0, "elem": 0.0, "chain": 0.0, "-": 0.0}
    for (role, name), c in zip(PHASES, buf):
        per = c / chunks
        tot[role] += per
        if role != "-":
            print(f"{role:5s}  {name:46s} {per:8.0f} cycles/chunk")
    print(f"aux {tot['aux']:.0f}, element {tot['elem']:.0f}, chain {tot['chain']:.0f} cycles/chunk")
    # per-CTA spans of the same launch: the kernel ends with its slowest CTA
    lib.kda_debug_pipe_cta.restype = ctypes.c_int
    nrec = 4 + len(PHASES)
    rec = (ctypes.c_ulonglong * (nrec * 1024))()
    n = lib.kda_debug_pipe_cta(rec, 1024)
    ctas = []
    for i in range(max(n, 0)):
        r = rec[nrec * i:nrec * (i + 1)]
        if r[1] > r[0] and r[2] > 0:
            ctas.append({"us": (r[1] - r[0]) / 1e3, "chunks": r[2], "sm": r[3], "t0": r[0], "ph": r[4:]})
    if ctas:
        ctas.sort(key=lambda c: c["us"])
        start = min(c["t0"] for c in ctas)
        per = sorted(c["us"] / c["chunks"] for c in ctas)
        print(f"CTAs {len(ctas)}: span min {ctas[0]['us']:.1f} median {ctas[len(ctas) // 2]['us']:.1f} "
              f"max {ctas[-1]['us']:.1f} us; us per chunk min {per[0]:.3f} median {per[len(per) // 2]:.3f} "
              f"max {per[-1]:.3f}; latest start {max(c['t0'] - start for c in ctas) / 1e3:.1f} us")
        by_rate = sorted(ctas, key=lambda c: c["us"] / c["chunks"])
        for label, group in (("fastest", by_rate[:8]), ("slowest", by_rate[-8:])):
            print(f"{label} 8 CTAs per chunk (us {sum(c['us'] / c['chunks'] for c in group) / 8:.3f}; "
                  f"SMs {[c['sm'] for c in group]}; chunks {[c['chunks'] for c in group]}):")
            for k, (role, name) in enumerate(PHASES):
                if role == "-":
                    continue
                v = sum(c["ph"][k] / c["chunks"] for c in group) / len(group)
                print(f"   {role:5s}  {name:46s} {v:8.0f}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
