"""Seeded synthetic workloads for the KDA chunked-prefill forward.

This module holds the workload definitions and the seeded input generators
and nothing of the method's arithmetic, so that both the oracle side
(tests, CPU baseline) and the CUDA side (tests, bench) can draw identical
inputs from it.

The shapes follow the H20 benchmark table of the FlashKDA release
(toolarium.ru post, section "Что показывают H20-бенчмарки": T=8192, D=128,
H in {96, 64}, fixed length, varlen seq_lens=[1300, 547, 2048, 963, 271, 3063]
and varlen 1024 x 8).  The pages give shapes only; the value distributions
below are synthetic stand-ins (no dataset is named):

  q, k  ~ N(0,1) fp32, L2-normalised per (token, head), then cast to bf16
  v     ~ N(0,1) -> bf16
  g     ~ N(0,1) fp32 (raw gate input)
  beta  = sigmoid(N(0,1)) fp32
  A_log = log U[1,16] per head (fp32)
  dt_bias ~ N(0, 0.1) per (head, channel) fp32
  lower_bound = -5, scale = 1/sqrt(128)
  initial state (where used) ~ N(0, 0.02) fp32, 0.02 read as the std.

Seeds: torch.Generator('cpu').manual_seed(1000 + workload id), drawing in the
fixed order q, k, v, g, beta, A_log, dt_bias, initial_state.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import torch

HEAD_DIM = 128


@dataclass(frozen=True)
class Workload:
    wid: int
    name: str
    H: int
    seq_lens: tuple              # one entry per sequence
    packed: bool                 # True: cu_seqlens layout; False: [B, T] fixed
    init: Optional[str]          # None (NULL state), "zero", "normal"
    final: bool                  # return the final state
    K: int = HEAD_DIM
    V: int = HEAD_DIM
    lower_bound: float = -5.0

    @property
    def T(self) -> int:
        return int(sum(self.seq_lens))

    @property
    def N(self) -> int:
        return len(self.seq_lens)

    @property
    def scale(self) -> float:
        return self.K ** -0.5

    def describe(self) -> str:
        if self.packed:
            lay = f"varlen seq_lens={list(self.seq_lens)}" if len(set(self.seq_lens)) > 1 \
                else f"varlen {self.seq_lens[0]}x{self.N}"
        else:
            lay = f"fixed B={self.N} T={self.seq_lens[0]}"
        st = {None: "no initial state", "zero": "zero initial state",
              "normal": "initial state N(0,0.02)"}[self.init]
        return (f"KDA prefill T={self.T} H={self.H} K=V={self.K} {lay}, {st}"
                + (", final state returned" if self.final else ""))


WORKLOADS = {
    0: Workload(0, "tiny_t256_h2", H=2, seq_lens=(256,), packed=False, init="zero", final=True),
    1: Workload(1, "fixed_t8192_h64", H=64, seq_lens=(8192,), packed=False, init=None, final=False),
    2: Workload(2, "varlen6_t8192_h96", H=96, seq_lens=(1300, 547, 2048, 963, 271, 3063),
                packed=True, init=None, final=False),
    3: Workload(3, "stateful_8x1024_h64", H=64, seq_lens=(1024,) * 8, packed=True,
                init="normal", final=True),
    4: Workload(4, "long_t131072_h32", H=32, seq_lens=(131072,), packed=False,
                init="normal", final=True),
}


def custom(seq_lens, H: int, *, packed: bool = True, init: Optional[str] = None,
           final: bool = True, lower_bound: float = -5.0, wid: int = 99,
           name: str = "custom") -> Workload:
    """A workload of arbitrary shape with the standard value distributions."""
    return Workload(wid, name, H=H, seq_lens=tuple(int(s) for s in seq_lens), packed=packed,
                    init=init, final=final, lower_bound=lower_bound)


def _l2n(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def make_inputs(w: Workload, seed: Optional[int] = None) -> dict:
    """Seeded CPU tensors for workload ``w`` in the packed [T, H, D] layout.

    Returns a dict with q, k, v (bf16), g (fp32 [T,H,K]), beta (fp32 [T,H]),
    A_log (fp32 [H]), dt_bias (fp32 [H,K]), lower_bound, scale,
    initial_state (fp32 [N,H,K,V] or None), cu_seqlens (int32 [N+1] or None),
    batch, seqlen and N.  For a fixed-length workload cu_seqlens is None and
    the tensors are the row-major flattening of [B, T, H, D].
    """
    gen = torch.Generator("cpu")
    gen.manual_seed(1000 + w.wid if seed is None else seed)
    T, H, K, V = w.T, w.H, w.K, w.V
    q = _l2n(torch.randn(T, H, K, generator=gen)).to(torch.bfloat16)
    k = _l2n(torch.randn(T, H, K, generator=gen)).to(torch.bfloat16)
    v = torch.randn(T, H, V, generator=gen).to(torch.bfloat16)
    g = torch.randn(T, H, K, generator=gen)
    beta = torch.sigmoid(torch.randn(T, H, generator=gen))
    A_log = torch.log(torch.empty(H).uniform_(1.0, 16.0, generator=gen))
    dt_bias = torch.randn(H, K, generator=gen) * 0.1
    init = None
    if w.init == "zero":
        init = torch.zeros(w.N, H, K, V)
    elif w.init == "normal":
        init = torch.randn(w.N, H, K, V, generator=gen) * 0.02
    cu = None
    if w.packed:
        offs = [0]
        for s in w.seq_lens:
            offs.append(offs[-1] + s)
        cu = torch.tensor(offs, dtype=torch.int32)
    return dict(q=q, k=k, v=v, g=g, beta=beta, A_log=A_log, dt_bias=dt_bias,
                lower_bound=float(w.lower_bound), scale=float(w.scale),
                initial_state=init, cu_seqlens=cu,
                batch=1 if w.packed else w.N,
                seqlen=w.T if w.packed else w.seq_lens[0], N=w.N)


def cotangents(w: Workload, seed: Optional[int] = None):
    """Seeded gradients of the forward's outputs for the backward: d_out (bf16 [T, H, V],
    standard normal) and d_final_state (fp32 [N, H, K, V], normal with std 0.1)."""
    gen = torch.Generator("cpu")
    gen.manual_seed(5000 + w.wid if seed is None else seed)
    d_out = torch.randn(w.T, w.H, w.V, generator=gen).to(torch.bfloat16)
    d_final = torch.randn(w.N, w.H, w.K, w.V, generator=gen) * 0.1
    return d_out, d_final


def gdn_inputs(x: dict) -> dict:
    """Inputs of the scalar-gate variant drawn from the same seeded tensors: the gate
    input and dt_bias of channel 0 (same distributions, one value per token-head / head)."""
    y = dict(x)
    y["g"] = x["g"][..., 0].contiguous()
    y["dt_bias"] = x["dt_bias"][:, 0].contiguous()
    return y
