#!/usr/bin/env python
"""KDA chunked-prefill throughput on B200 (one JSON line on stdout).

Workload (default): T = 8192 packed tokens, seq_lens [1300, 547, 2048, 963, 271,
3063], H = 96, K = V = 128, bf16 q/k/v, fp32 gates, no initial state -- the
varlen row of the FlashKDA H20 benchmark table (toolarium.ru post, section
"Что показывают H20-бенчмарки"), with synthetic seeded inputs (kda_workloads).

A step is one kda_fwd call over the whole batch (the fused tcgen05 kernel:
gate pre-pass, intra-chunk WY, state propagation and output in one launch).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kda|reference]

With N > 1 (torchrun, one rank per GPU) every rank runs an independent
replica of the workload (the forward has no cross-GPU exchange); the value is
the tokens of all ranks over the slowest rank's time.  --impl reference times
the fp64 CPU oracle on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import kda_workloads as W  # noqa: E402

BYTES_PER_TOKEN_HEAD = 1540          # q,k,v bf16 768 + g fp32 512 + beta 4 + out bf16 256
STATE_BYTES = 128 * 128 * 4          # one (sequence, head) state, read or written
FLOP_PER_TOKEN_HEAD = 180224         # 10 C D + 6 D^2 with C = 64, D = 128
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0             # the spec sheet's HBM3e figure, for context
NOMINAL_BF16_TFLOPS = 2250.0         # dense bf16 tensor peak, spec sheet, for context


def workload(args) -> "W.Workload":
    """The workload of --workload, with --heads applied (same sequences, seed and values)."""
    import dataclasses
    w = W.WORKLOADS[args.workload]
    if args.heads:
        w = dataclasses.replace(w, H=args.heads, name=f"{w.name}_h{args.heads}")
    if args.lower_bound is not None:
        w = dataclasses.replace(w, lower_bound=args.lower_bound, name=f"{w.name}_lb{args.lower_bound:g}")
    return w


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["kda", "reference"], default="kda")
    ap.add_argument("--workload", type=int, default=2, choices=sorted(W.WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--gdn", action="store_true",
                    help="time kda_gdn_fwd, the scalar-gate variant, on the same workload")
    ap.add_argument("--decode", action="store_true",
                    help="time kda_decode (one token per sequence) instead of the prefill")
    ap.add_argument("--bwd", action="store_true",
                    help="time the backward kda_bwd (all gradients) instead of the forward")
    ap.add_argument("--lower-bound", type=float, default=None,
                    help="override the workload's gate clamp (below -9.5 kda_fwd takes the staged kernels)")
    ap.add_argument("--heads", type=int, default=0,
                    help="override the workload's head count (small cases for profiling)")
    ap.add_argument("--segments", type=int, default=0,
                    help="one-sequence workloads: run the forward as R segments per pass "
                         "(cp.segmented_prefill) instead of one kda_fwd call; -1 = cp.choose_segments")
    ap.add_argument("--decode-batch", type=int, default=256)
    ap.add_argument("--decode-heads", type=int, default=96)
    return ap.parse_args()


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_bf16_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return 1590.0


GDN_BYTES_PER_TOKEN_HEAD = 1032    # q,k,v bf16 768 + g fp32 4 + beta 4 + out bf16 256


def algorithmic_bytes(w: W.Workload, gdn: bool = False) -> int:
    b = (GDN_BYTES_PER_TOKEN_HEAD if gdn else BYTES_PER_TOKEN_HEAD) * w.T * w.H
    if w.init is not None:
        b += STATE_BYTES * w.N * w.H
    if w.final:
        b += STATE_BYTES * w.N * w.H
    return b


KERNEL_SOURCES = {
    "kda_pipe_kernel": ("kda_pipe.cuh", "umma.cuh", "warp_mma.cuh", "kda_common.cuh"),
    "kda_pipe_kernel<scalar gate>": ("kda_pipe.cuh", "umma.cuh", "warp_mma.cuh", "kda_common.cuh"),
    "kda_decode_kernel": ("kda_decode.cuh", "kda_common.cuh"),
}


def kernel_source_hash(kernel: str = "kda_pipe_kernel") -> str:
    """Hash of the device sources one kernel is compiled from (profiles carry it
    so that stale DRAM counters are not reported against a changed kernel)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_delta_rule_135_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


TRAFFIC_FILES = {"kda_pipe_kernel": "kda_pipe_traffic.json",
                 "kda_pipe_kernel<scalar gate>": "kda_gdn_traffic.json",
                 "kda_decode_kernel": "kda_decode_traffic.json"}


def dram_traffic_from_profile(kernel: str, units: float):
    """Per-launch DRAM bytes (read + write) of ``kernel`` from its committed ncu
    summary, scaled to ``units`` (token-heads for the prefill, sequence-heads
    for decode), if the counters were taken on the current kernel source; else
    None."""
    path = os.path.join(ROOT, "profiles", TRAFFIC_FILES[kernel])
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("kernel_source_hash") != kernel_source_hash(kernel):
        return None
    per_unit = d.get("dram_bytes_per_unit")
    if per_unit is None:
        return None
    return float(per_unit) * units


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x0000000000000004: "sw_power_cap",
        0x0000000000000008: "hw_slowdown",
        0x0000000000000020: "sw_thermal_slowdown",
        0x0000000000000040: "hw_thermal_slowdown",
        0x0000000000000080: "hw_power_brake_slowdown",
    }

    def __init__(self, device_index: int):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            pass

    def sample(self):
        if not self._ok:
            return
        nv = self.nv
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
            mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for bit, name in self.REASONS.items():
                if mask & bit:
                    self.reasons.add(name)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self.sample()
            time.sleep(0.002)

    def wait(self, event):
        """Samples from the calling thread until ``event`` has completed (the
        launches are queued already, so the GPU stays busy meanwhile)."""
        while not event.query():
            self.sample()
            time.sleep(0.0005)
        torch.cuda.synchronize()

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self._ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if args.impl == "kda" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available() and args.impl == "kda":
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def oracle_sample(w: W.Workload, x: dict, target_s: float, gdn: bool = False):
    """Runs the fp64 oracle on the first h heads of every sequence, h sized so
    the run takes about target_s seconds; returns (tokens-equivalent/s, desc)."""
    import oracle
    cores = len(os.sched_getaffinity(0))

    def run(h):
        sub = dict(x)
        for key in ("q", "k", "v", "g", "beta"):
            sub[key] = x[key][:, :h].contiguous()
        sub["A_log"] = x["A_log"][:h]
        sub["dt_bias"] = x["dt_bias"][:h]
        fwd = oracle.gdn_recurrent if gdn else oracle.recurrent
        if x["initial_state"] is not None:
            sub["initial_state"] = x["initial_state"][:, :h].contiguous()
        t = time.perf_counter()
        fwd(sub["q"], sub["k"], sub["v"], sub["g"], sub["beta"], sub["A_log"],
                         sub["dt_bias"], sub["lower_bound"], sub["scale"], sub["initial_state"],
                         sub["cu_seqlens"], want_final=w.final)
        return time.perf_counter() - t

    # calibrate on one head: its N (sequence, head) units run on min(N, cores) threads
    t1 = run(1)
    per_token_head = t1 * min(w.N, cores) / w.T          # core-seconds per token-head
    h = int(target_s * cores / max(per_token_head * w.T, 1e-9))
    h = max(1, min(w.H, h))
    t = run(h) if h > 1 else t1
    rate = (w.T * h / w.H) / t          # whole-workload tokens per second equivalent
    desc = (f"oracle over heads 0..{h - 1} of {w.H} (all {w.N} sequences, {w.T * h} token-heads) "
            f"in {t:.2f} s on {oracle.max_threads()} OpenMP threads; scaled by {h}/{w.H}")
    return rate, desc, cores, oracle.max_threads(), h


def workload_config(w: W.Workload, world: int, parallelism: str, gdn: bool = False, segments: int = 0) -> dict:
    """The `config` object of a bench line: the workload and its sizes (the same keys on every
    arm, so that lines of the same workload compare)."""
    return {"workload": ("GDN (one gate per token-head) " if gdn else "") + w.describe()
                        + (f"; run as {segments} segments (maps, fold, final pass)" if segments else ""),
            "global_batch": w.N * world, "seq_len": w.T, "heads": w.H,
            "parallelism": parallelism,
            "l2": f"inputs exceed L2 ({algorithmic_bytes(w, gdn) / 1e6:.0f} MB per step vs 126 MB); no flush"}


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    w = workload(args)
    x = W.make_inputs(w)
    import oracle
    # size each step's sample so the whole run stays within a few minutes
    per_step_target = max(0.5, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    rate, desc, cores, threads, h = oracle_sample(w, x, per_step_target)

    def step():
        sub = dict(x)
        for key in ("q", "k", "v", "g", "beta"):
            sub[key] = x[key][:, :h].contiguous()
        sub["A_log"] = x["A_log"][:h]
        sub["dt_bias"] = x["dt_bias"][:h]
        if x["initial_state"] is not None:
            sub["initial_state"] = x["initial_state"][:, :h].contiguous()
        oracle.recurrent(sub["q"], sub["k"], sub["v"], sub["g"], sub["beta"], sub["A_log"],
                         sub["dt_bias"], sub["lower_bound"], sub["scale"], sub["initial_state"],
                         sub["cu_seqlens"], want_final=w.final)

    for _ in range(args.warmup):
        step()
    t = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t
    ms_per_step = el / args.steps * 1e3 * (w.H / h)     # whole-workload equivalent
    value = w.T / (ms_per_step / 1e3) / 1e6
    line = {
        "impl": "reference", "metric": "KDA prefill throughput (Mtokens/s) at T=8192 H=96 D=128 varlen",
        "value": value, "unit": "Mtokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, world, "host cores (OpenMP over sequence x head)"),
        "precision": "fp64 token-by-token recurrence (the oracle)",
        "cpu_baseline": {"value": value, "unit": "Mtokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"each step: {desc.split(' in ')[0]}; scaled by {h}/{w.H}"},
        "e2e": {"value": value, "unit": "Mtokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


DECODE_BYTES_PER_SEQ_HEAD = 2 * STATE_BYTES + 768 + 512 + 4 + 256   # state in + out, q/k/v, g, beta, o


def run_decode(args, world, rank, kda):
    """kda_decode over B sequences x H heads per step: one token each, the fp32
    states updated in place (B H 128 KiB of state traffic per step)."""
    B, H = args.decode_batch, args.decode_heads
    gen = torch.Generator("cpu").manual_seed(2000)
    dev = torch.device("cuda", torch.cuda.current_device())
    w = W.custom([1] * B, H=H, packed=False, init="normal", wid=60)
    x = W.make_inputs(w)
    xd = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    state = (torch.randn(B, H, 128, 128, generator=gen) * 0.02).to(dev)
    out = torch.empty(B, H, 128, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        kda.kda_decode(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"],
                       x["lower_bound"], x["scale"], state, out=out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if kda.kda_check_device_error() != 0:
        raise RuntimeError("device error recorded during warm-up")
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(dev.index)
    barrier(world)
    torch.cuda.synchronize()
    with sampler:
        for i in range(args.steps):
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        sampler.wait(ends[-1])
    barrier(world)
    kernel_ms = statistics.mean(s.elapsed_time(e) for s, e in zip(starts, ends))
    total_ms = max_over_ranks(starts[0].elapsed_time(ends[-1]), world)
    ms_per_step = total_ms / args.steps
    value = B * world / (ms_per_step / 1e3) / 1e6
    alg_bytes = DECODE_BYTES_PER_SEQ_HEAD * B * H
    peak, peak_kind = measured_hbm_peak()
    achieved = alg_bytes / (kernel_ms / 1e3) / 1e9

    e2e = None
    if args.e2e_steps > 0:
        keys = ("q", "k", "v", "g", "beta")
        host = {k: x[k].pin_memory() for k in keys}
        out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(host[k].numel() * host[k].element_size() for k in keys)
        d2h = out_h.numel() * out_h.element_size()
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            for k in keys:
                xd[k].copy_(host[k], non_blocking=True)
            step()
            out_h.copy_(out, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1), world) / args.e2e_steps
        e2e = {"value": B * world / (e_ms / 1e3) / 1e6, "unit": "Mtokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        sub_b = max(1, min(B, 32))
        xs = {k: x[k][:sub_b] for k in ("q", "k", "v", "g", "beta")}
        st = state[:sub_b].cpu()
        t = time.perf_counter()
        oracle.recurrent(xs["q"], xs["k"], xs["v"], xs["g"], xs["beta"], x["A_log"], x["dt_bias"],
                         x["lower_bound"], x["scale"], st, oracle.fixed_offsets(sub_b, 1))
        el = time.perf_counter() - t
        cpu = {"value": sub_b / el / 1e6, "unit": "Mtokens/s", "cores": oracle.max_threads(),
               "kind": "oracle", "sample": f"{sub_b} of {B} sequences x {H} heads, one token each"}

    if rank == 0:
        line = {
            "metric": f"KDA decode throughput (Mtokens/s) at B={B} H={H} D=128",
            "value": value, "unit": "Mtokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded kda_workloads, no dataset)",
            "config": {"workload": f"decode B={B} H={H} K=V=128, fp32 state in place",
                       "global_batch": B * world, "seq_len": 1, "heads": H,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": f"state {B * H * STATE_BYTES / 1e9:.2f} GB exceeds L2; no flush"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak,
                         "traffic": dram_traffic_from_profile("kda_decode_kernel", B * H),
                         "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)",
                         "kernel": "kda_decode_kernel", "kernel_ms": kernel_ms,
                         "algorithmic_bytes": alg_bytes},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps,
            "clocks": sampler.summary(),
        }
        print(json.dumps(line), flush=True)
    return 0


BWD_BYTES_PER_TOKEN_HEAD = 3592   # reads q,k,v bf16 768, g 512, beta 4, d_out bf16 256; writes dq,dk,dv,dg fp32 2048, dbeta 4
BWD_LAUNCHES_PER_STEP = 9         # staged forward 4 (no output kernel) + backward 5


def run_backward(args, world, rank, kda):
    """kda_bwd over the workload: every gradient (dq, dk, dv, dg, dbeta, dA_log, ddt_bias
    and the initial-state gradient when the workload has states) per step."""
    w = workload(args)
    x = W.make_inputs(w)
    dO, dF = W.cotangents(w)
    if not w.final:
        dF = None
    dev = torch.device("cuda", torch.cuda.current_device())
    xd = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    dOd = dO.to(dev)
    dFd = dF.to(dev) if dF is not None else None
    want_dinit = w.init is not None
    grads = kda.kda_bwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"],
                        x["lower_bound"], x["scale"], dOd, xd["initial_state"], xd["cu_seqlens"], dFd,
                        want_d_initial=want_dinit, batch=x["batch"])
    ws = torch.empty(kda.kda_bwd_workspace_size(xd["q"], xd["cu_seqlens"], x["batch"]), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream()

    def step():
        kda.kda_bwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"],
                    x["lower_bound"], x["scale"], dOd, xd["initial_state"], xd["cu_seqlens"], dFd,
                    want_d_initial=want_dinit, grads=grads, workspace=ws, batch=x["batch"])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if kda.kda_check_device_error() != 0:
        raise RuntimeError("device error recorded during warm-up")
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(dev.index)
    barrier(world)
    torch.cuda.synchronize()
    with sampler:
        for i in range(args.steps):
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        sampler.wait(ends[-1])
    barrier(world)
    step_ms = statistics.mean(s.elapsed_time(e) for s, e in zip(starts, ends))
    total_ms = max_over_ranks(starts[0].elapsed_time(ends[-1]), world)
    ms_per_step = total_ms / args.steps
    value = w.T * world / (ms_per_step / 1e3) / 1e6
    alg_bytes = BWD_BYTES_PER_TOKEN_HEAD * w.T * w.H + STATE_BYTES * w.N * w.H * (
        (w.init is not None) + (dF is not None) + want_dinit)
    peak, peak_kind = measured_hbm_peak()
    achieved = alg_bytes / (step_ms / 1e3) / 1e9

    e2e = None
    if args.e2e_steps > 0:
        keys = ("q", "k", "v", "g", "beta")
        host = {k: x[k].pin_memory() for k in keys}
        dO_h = dO.pin_memory()
        outs = ("dq", "dk", "dv", "dg", "dbeta")
        out_h = {n: torch.empty(grads[n].shape, dtype=grads[n].dtype).pin_memory() for n in outs}
        h2d = sum(host[k].numel() * host[k].element_size() for k in keys) + dO_h.numel() * dO_h.element_size()
        d2h = sum(t.numel() * t.element_size() for t in out_h.values())
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            for k in keys:
                xd[k].copy_(host[k], non_blocking=True)
            dOd.copy_(dO_h, non_blocking=True)
            step()
            for n in outs:
                out_h[n].copy_(grads[n], non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1), world) / args.e2e_steps
        e2e = {"value": w.T * world / (e_ms / 1e3) / 1e6, "unit": "Mtokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from threadpoolctl import threadpool_limits
        from oracle import backward as OB
        h = max(1, min(w.H, int(args.cpu_seconds / 4.0)))     # about 4 s of oracle per head at T = 8192
        sub = {key: x[key][:, :h].contiguous() for key in ("q", "k", "v", "g", "beta")}
        init = x["initial_state"][:, :h].contiguous() if x["initial_state"] is not None else None
        dsub = dF[:, :h].contiguous() if dF is not None else None
        cu = x["cu_seqlens"] if x["cu_seqlens"] is not None else \
            torch.arange(x["batch"] + 1, dtype=torch.int32) * x["seqlen"]
        with threadpool_limits(1):
            t = time.perf_counter()
            OB.grads_chunked(sub["q"], sub["k"], sub["v"], sub["g"], sub["beta"], x["A_log"][:h],
                             x["dt_bias"][:h], x["lower_bound"], x["scale"], init, cu,
                             dO[:, :h].contiguous(), dsub)
            el = time.perf_counter() - t
        cpu = {"value": (w.T * h / w.H) / el / 1e6, "unit": "Mtokens/s", "cores": 1, "kind": "oracle",
               "sample": f"chunked fp64 backward oracle over heads 0..{h - 1} of {w.H} ({w.T * h} token-heads) "
                         f"in {el:.2f} s on one thread; scaled by {h}/{w.H}"}

    if rank == 0:
        line = {
            "metric": "KDA backward throughput (Mtokens/s) at T=8192 H=96 D=128 varlen"
            if args.workload == 2 else f"KDA backward throughput (Mtokens/s), {w.name}",
            "value": value, "unit": "Mtokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded kda_workloads, no dataset)",
            "config": {"workload": "backward (all gradients) of " + w.describe(),
                       "model": "KDA layer backward (no weights)",
                       "global_batch": w.N * world, "seq_len": w.T, "heads": w.H,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "precision": "bf16 q/k/v/d_out, fp32 gates, states and gradients; fp32 CUDA cores",
                       "l2": f"inputs and gradients exceed L2 ({alg_bytes / 1e6:.0f} MB per step); no flush"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": None,
                         "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)",
                         "kernel": f"whole backward step ({BWD_LAUNCHES_PER_STEP} launches)",
                         "kernel_ms": step_ms, "algorithmic_bytes": alg_bytes},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": BWD_LAUNCHES_PER_STEP * args.steps,
            "clocks": sampler.summary(),
        }
        print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    assert args.warmup >= 3, "at least 3 warm-up steps"
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        rc = run_reference(args, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return rc

    import kda_build as build
    if rank == 0:
        build.build()
    barrier(world)
    import gated_delta_rule_135_b200 as kda
    if args.decode or args.bwd:
        rc = (run_decode if args.decode else run_backward)(args, world, rank, kda)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return rc

    w = workload(args)
    x = W.make_inputs(w)
    if args.gdn:
        x = W.gdn_inputs(x)
    dev = torch.device("cuda", torch.cuda.current_device())
    xd = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    out = torch.empty_like(xd["q"])
    fin = (torch.empty(w.N, w.H, 128, 128, device=dev) if w.final else None)
    stream = torch.cuda.current_stream()
    fused = args.gdn or x["lower_bound"] >= kda.FUSED_MIN_LOWER_BOUND
    launches_per_step = 1 if fused else 5
    # one long sequence in the fixed layout: the library splits it into segments itself
    lib_segments = (kda.kda_fwd_segments(w.H, w.T) if fused and w.N == 1 and x["cu_seqlens"] is None else 1)
    if lib_segments > 1:
        launches_per_step = lib_segments + 3   # segment offsets, two map passes, R - 1 folds, final pass
    fwd = kda.kda_gdn_fwd if args.gdn else kda.kda_fwd
    seg_ws = {}
    if args.segments:
        assert w.N == 1 and fused, "--segments takes a one-sequence workload on the fused path"
        from gated_delta_rule_135_b200 import cp
        from gated_delta_rule_135_b200.cp import choose_segments, segment_offsets
        if args.segments < 0:     # the library's choice
            args.segments = choose_segments(w.T, w.H, torch.cuda.get_device_properties(dev).multi_processor_count)
        n_seg = len(segment_offsets(w.T, args.segments)) - 1
        launches_per_step = 1 if n_seg == 1 else 3 + (n_seg - 1)

    def step():
        if args.segments:
            o, f = cp.segmented_prefill(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"],
                                        xd["dt_bias"], x["lower_bound"], x["scale"], xd["initial_state"],
                                        segments=args.segments, gdn=args.gdn, out=out, workspace=seg_ws)
            return
        fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"],
            x["lower_bound"], x["scale"], xd["initial_state"], xd["cu_seqlens"], out=out,
            final_state=fin, batch=x["batch"])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if kda.kda_check_device_error() != 0:
        raise RuntimeError("device error recorded during warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(dev.index)
    barrier(world)
    torch.cuda.synchronize()
    with sampler:
        for i in range(args.steps):
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        sampler.wait(ends[-1])
    barrier(world)
    per_step = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = starts[0].elapsed_time(ends[-1])
    total_ms = max_over_ranks(total_ms, world)
    ms_per_step = total_ms / args.steps
    tokens = w.T * world
    value = tokens / (ms_per_step / 1e3) / 1e6
    tflops = FLOP_PER_TOKEN_HEAD * w.T * w.H * world / (ms_per_step / 1e3) / 1e12
    kernel_ms = statistics.mean(per_step)
    alg_bytes = algorithmic_bytes(w, args.gdn)
    peak, peak_kind = measured_hbm_peak()
    achieved = alg_bytes / (kernel_ms / 1e3) / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak,
            "traffic": (dram_traffic_from_profile("kda_pipe_kernel<scalar gate>" if args.gdn else "kda_pipe_kernel",
                                                  w.T * w.H)
                        if fused and not args.segments and lib_segments == 1 else None),
            "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)" if peak_kind == "measured"
            else "fallback 6650 GB/s",
            "kernel": (f"segmented prefill ({args.segments} segments: 3 fused launches + folds)" if args.segments
                       else (f"{fwd.__name__} split into {lib_segments} segments by the library (3 fused launches "
                             f"+ folds)") if lib_segments > 1
                       else ("kda_pipe_kernel<scalar gate>" if args.gdn else "kda_pipe_kernel") if fused
                       else "staged kernels"),
            "kernel_ms": kernel_ms, "algorithmic_bytes": alg_bytes,
            "tflops": tflops,
            "frac_nominal_hbm": achieved / NOMINAL_HBM_GBS,
            "tensor": {"achieved_tflops": tflops, "peak_tflops": measured_bf16_peak(),
                       "frac": tflops / measured_bf16_peak(),
                       "frac_nominal": tflops / NOMINAL_BF16_TFLOPS,
                       "flop_per_token_head": FLOP_PER_TOKEN_HEAD}}

    # end to end through the public API with host buffers
    e2e = None
    if args.e2e_steps > 0:
        keys = ("q", "k", "v", "g", "beta")
        host = {k: x[k].pin_memory() for k in keys}
        out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(host[k].numel() * host[k].element_size() for k in keys)
        d2h = out_h.numel() * out_h.element_size()
        for _ in range(2):
            for k in keys:
                xd[k].copy_(host[k], non_blocking=True)
            step()
            out_h.copy_(out, non_blocking=True)
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            for k in keys:
                xd[k].copy_(host[k], non_blocking=True)
            step()
            out_h.copy_(out, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1), world) / args.e2e_steps
        e2e = {"value": tokens / (e_ms / 1e3) / 1e6, "unit": "Mtokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, desc, cores, threads, _ = oracle_sample(w, x, args.cpu_seconds, args.gdn)
        cpu = {"value": rate / 1e6, "unit": "Mtokens/s", "cores": threads, "kind": "oracle",
               "sample": desc, "host_cores": cores}

    if rank == 0:
        line = {
            "metric": (("GDN (scalar-gate) prefill throughput (Mtokens/s) at T=8192 H=96 D=128 varlen"
                        if args.gdn else "KDA prefill throughput (Mtokens/s) at T=8192 H=96 D=128 varlen")
                       if args.workload == 2 and not args.heads and args.lower_bound is None else
                       f"{'GDN (scalar-gate)' if args.gdn else 'KDA'} prefill throughput (Mtokens/s), {w.name}"),
            "value": value, "unit": "Mtokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded kda_workloads, no dataset)",
            "config": workload_config(w, world, f"replicas x{world}" if world > 1 else "single GPU",
                                      args.gdn, args.segments),
            "precision": "bf16 q/k/v/out, fp32 gates and state; bf16/fp16 MMA operands, fp32 accumulate",
            "tflops": tflops,
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": sampler.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
