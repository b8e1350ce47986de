"""Context-parallel prefill of one long sequence over the ranks of a process group.

The KDA (and scalar-gate) recurrence is affine in the state a segment starts from:
after a segment, S_out = A S_in + B.  Here A is the segment's final state from S_in = I
with v = 0, and B its final state from S_in = 0.  Each rank holds one contiguous segment
and:

1. runs the forward twice on its segment to get (A_r, B_r);
2. all-gathers every rank's (A_r, B_r);
3. folds S_r = A_{r-1}(... (A_0 S_0 + B_0) ...) + B_{r-1} with kda_state_affine;
4. runs the forward on its segment from S_r, which gives its outputs and (on the last
   rank) the sequence's final state.

That is three forward passes over T / R tokens per rank, so about R / 3 times faster than
one GPU for long sequences.  The exchange carries 2 x 64 KiB per head and rank.  The
FlashKDA posts motivate long-context prefill (128k-1M tokens; donniechu.com, section "Số
liệu kỹ thuật").

Host plumbing only: the forwards and the fold run in the library's kernels.  ``fwd`` and
``affine`` can be replaced (tests drive the same steps with the fp64 oracle on CPU ranks).
"""
from __future__ import annotations

from typing import Callable, Optional

import torch
import torch.distributed as dist

HEAD_DIM = 128


def segment_maps(fwd: Callable, q, k, v, g, beta, A_log, dt_bias, lower_bound: float, scale: float):
    """(A, B) of one segment, stacked as [2, H, 128, 128] fp32."""
    H = q.shape[-2]
    eye = torch.eye(HEAD_DIM, dtype=torch.float32, device=q.device).expand(1, H, HEAD_DIM, HEAD_DIM).contiguous()
    AB = torch.empty(2, H, HEAD_DIM, HEAD_DIM, dtype=torch.float32, device=q.device)
    fwd(q, k, torch.zeros_like(v), g, beta, A_log, dt_bias, lower_bound, scale, eye, None,
        final_state=AB[0:1])
    fwd(q, k, v, g, beta, A_log, dt_bias, lower_bound, scale, None, None, final_state=AB[1:2])
    return AB


def fold(affine: Callable, maps: torch.Tensor, initial_state: Optional[torch.Tensor], upto: int,
         H: int, device) -> torch.Tensor:
    """The state segment ``upto`` starts from: S_0 = initial_state (zeros if None), then
    S <- A_r S + B_r for r < upto.  maps: [R, 2, H, 128, 128]."""
    S = (torch.zeros(1, H, HEAD_DIM, HEAD_DIM, dtype=torch.float32, device=device)
         if initial_state is None else initial_state.reshape(1, H, HEAD_DIM, HEAD_DIM).contiguous())
    for r in range(upto):
        S = affine(maps[r, 0].contiguous(), S, maps[r, 1].contiguous()).reshape(1, H, HEAD_DIM, HEAD_DIM)
    return S


def cp_prefill(q, k, v, g, beta, A_log, dt_bias, lower_bound: float, scale: float,
               initial_state: Optional[torch.Tensor] = None, *, group=None, gdn: bool = False,
               fwd: Optional[Callable] = None, affine: Optional[Callable] = None):
    """Context-parallel forward of one sequence.  Each rank passes its own contiguous
    segment: q, k, v [T_r, H, 128] bf16; g [T_r, H, 128] fp32 ([T_r, H] with gdn=True);
    beta [T_r, H].  The same A_log, dt_bias, lower_bound, scale and initial_state ([1, H,
    128, 128] fp32 or None) on every rank.  Returns (out_r [T_r, H, 128] bf16,
    final_state [1, H, 128, 128]).  On the last rank that final state is the sequence's.
    """
    if fwd is None or affine is None:
        import gated_delta_rule_135_b200 as kda   # the CUDA library; fails loudly if missing
        fwd = fwd or (kda.kda_gdn_fwd if gdn else kda.kda_fwd)
        affine = affine or kda.kda_state_affine
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    H = q.shape[-2]
    AB = segment_maps(fwd, q, k, v, g, beta, A_log, dt_bias, lower_bound, scale)
    parts = [torch.empty_like(AB) for _ in range(world)]
    dist.all_gather(parts, AB, group=group)
    maps = torch.stack(parts)
    S = fold(affine, maps, initial_state, rank, H, q.device)
    fin = torch.empty(1, H, HEAD_DIM, HEAD_DIM, dtype=torch.float32, device=q.device)
    out, fin = fwd(q, k, v, g, beta, A_log, dt_bias, lower_bound, scale, S, None, final_state=fin)
    return out, fin


def segment_offsets(T: int, segments: int, align: int = 64):
    """Boundaries of ``segments`` contiguous pieces of T tokens, at multiples of ``align``
    (the chunk), as a list [0, ..., T]; empty pieces are dropped."""
    step = -(-T // segments)
    step = -(-step // align) * align
    cuts = list(range(0, T, step)) + [T]
    return [c for i, c in enumerate(cuts) if i == 0 or c > cuts[i - 1]]


def choose_segments(T: int, H: int, n_sm: int, max_segments: int = 64, fold_cost: float = 0.6) -> int:
    """The segment count for segmented_prefill: the forward runs one CTA per (segment, head)
    and a CTA takes its units in turn, so a pass costs about ceil(R H / n_sm) rounds of
    ceil(T / R / 64) chunks; segments take three passes (one without), and each fold step
    costs about ``fold_cost`` chunk-times.  Returns the R of least estimated time (1 = run
    the plain forward)."""
    def cost(R):
        cuts = segment_offsets(T, R)
        R_eff = len(cuts) - 1
        longest = max(b - a for a, b in zip(cuts, cuts[1:]))
        rounds = -(-R_eff * H // n_sm)
        passes = 1 if R_eff == 1 else 3
        return passes * rounds * -(-longest // 64) + fold_cost * (R_eff - 1)
    best = min(range(1, max_segments + 1), key=lambda R: (cost(R), R))
    return len(segment_offsets(T, best)) - 1


def segmented_prefill(q, k, v, g, beta, A_log, dt_bias, lower_bound: float, scale: float,
                      initial_state: Optional[torch.Tensor] = None, *, segments: int = 0, gdn: bool = False,
                      out: Optional[torch.Tensor] = None, workspace: Optional[dict] = None):
    """The context-parallel decomposition on one GPU, for one sequence with few heads.

    The forward runs one CTA per (sequence, head), so a single long sequence keeps only H
    SMs busy.  Splitting it into R segments and running all segments as one varlen batch
    keeps R x H busy, at the price of three passes instead of one: (1) every segment from
    S = I with v = 0 gives its A map and (2) from S = 0 its B map, (3) the maps are folded
    into each segment's starting state with kda_state_affine, and (4) every segment runs
    from its state.  q, k, v [T, H, 128] bf16, g [T, H, 128] ([T, H] with gdn), beta [T, H];
    initial_state [1, H, 128, 128] or None.  Returns (out [T, H, 128] bf16, final_state
    [1, H, 128, 128]); ``out`` may supply the output buffer.  segments = 0 picks the count
    with choose_segments (1 runs the plain forward).  ``workspace`` (a dict) caches the offsets, the zero values, the
    identity states and the state buffers between calls of the same shape."""
    import gated_delta_rule_135_b200 as kda   # the CUDA library; fails loudly if missing
    fwd = kda.kda_gdn_fwd if gdn else kda.kda_fwd
    T, H = q.shape[0], q.shape[-2]
    dev = q.device
    if not segments:
        segments = choose_segments(T, H, torch.cuda.get_device_properties(dev).multi_processor_count)
    if segments == 1:
        fin = torch.empty(1, H, HEAD_DIM, HEAD_DIM, dtype=torch.float32, device=dev)
        return fwd(q, k, v, g, beta, A_log, dt_bias, lower_bound, scale, initial_state, None, out=out,
                   final_state=fin)
    ws = workspace if workspace is not None else {}
    key = (T, H, segments, str(dev))
    if ws.get("key") != key:
        cuts = segment_offsets(T, segments)
        R = len(cuts) - 1
        ws.clear()
        ws.update(key=key, R=R, cu=torch.tensor(cuts, dtype=torch.int32, device=dev),
                  zeros=torch.zeros_like(v),
                  eye=torch.eye(HEAD_DIM, dtype=torch.float32, device=dev).expand(R, H, HEAD_DIM, HEAD_DIM)
                  .contiguous(),
                  A=torch.empty(R, H, HEAD_DIM, HEAD_DIM, dtype=torch.float32, device=dev),
                  B=torch.empty(R, H, HEAD_DIM, HEAD_DIM, dtype=torch.float32, device=dev),
                  S=torch.empty(R, H, HEAD_DIM, HEAD_DIM, dtype=torch.float32, device=dev),
                  F=torch.empty(R, H, HEAD_DIM, HEAD_DIM, dtype=torch.float32, device=dev))
    R, cu = ws["R"], ws["cu"]
    fwd(q, k, ws["zeros"], g, beta, A_log, dt_bias, lower_bound, scale, ws["eye"], cu, final_state=ws["A"])
    out, _ = fwd(q, k, v, g, beta, A_log, dt_bias, lower_bound, scale, None, cu, out=out, final_state=ws["B"])
    S = ws["S"]
    if initial_state is None:
        S[0].zero_()
    else:
        S[0].copy_(initial_state.reshape(H, HEAD_DIM, HEAD_DIM))
    for r in range(1, R):
        kda.kda_state_affine(ws["A"][r - 1], S[r - 1], ws["B"][r - 1], out=S[r])
    out, _ = fwd(q, k, v, g, beta, A_log, dt_bias, lower_bound, scale, S, cu, out=out, final_state=ws["F"])
    return out, ws["F"][R - 1:R]
