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
