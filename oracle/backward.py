"""fp64 oracle of the KDA backward (gradients of the forward) -- TEST INFRASTRUCTURE.

Only tests/ and the CPU-baseline leg of bench.py may use it; it shares no code with the
CUDA library.  Two independent forms:

* ``grads_autograd``: PyTorch autograd through a token-by-token fp64 forward written in
  plain torch ops (the recurrence of kda_ref.c, all heads at once).  Its forward is
  checked against the C oracle and its gradients against finite differences.
* ``grads_chunked``: the chunked backward in numpy fp64, the chain rule taken by hand
  through the WY / UT form of the chunked forward (``chunk_step_bwd``, one chunk); it
  spells out each stage the GPU backward computes and agrees with autograd to ~1e-10.

The loss is L = <dO, out> + <dS_final, final_state>; every function returns
dq, dk, dv, dg, dbeta, dA_log, ddt_bias, dS0 (fp64 numpy).
"""
from __future__ import annotations

import numpy as np
import torch

from . import bf16_to_f64, _f32, _f64, _offsets, gate_np


def _t(x):
    return torch.as_tensor(np.asarray(x), dtype=torch.float64)


def forward_torch(q, k, v, g, beta, A_log, dt_bias, lower_bound: float, scale: float, S0, cu):
    """Token-by-token forward in torch fp64 (all heads per step).  q, k, v, g: [T, H, *];
    beta [T, H]; A_log [H]; dt_bias [H, K]; S0 [N, H, K, V]; cu: [N + 1] offsets."""
    T, H, K = q.shape
    la = torch.clamp_min(-torch.exp(A_log)[None, :, None] * torch.nn.functional.softplus(g + dt_bias[None]),
                         lower_bound)
    a = torch.exp(la)
    outs, fins = [], []
    for n in range(len(cu) - 1):
        S = S0[n]
        for t in range(int(cu[n]), int(cu[n + 1])):
            St = a[t][:, :, None] * S                                   # Diag(a) S
            e = v[t] - torch.einsum("hkv,hk->hv", St, k[t])            # v - S~^T k
            S = St + beta[t][:, None, None] * k[t][:, :, None] * e[:, None, :]
            outs.append(scale * torch.einsum("hkv,hk->hv", S, q[t]))
        fins.append(S)
    return torch.stack(outs) if outs else torch.zeros(0, H, v.shape[-1], dtype=torch.float64), torch.stack(fins)


def _inputs(q, k, v, g, beta, A_log, dt_bias, initial_state, cu_seqlens):
    qf, kf, vf = (_t(bf16_to_f64(x)) for x in (q, k, v))
    H, K = qf.shape[-2], qf.shape[-1]
    qf, kf, vf = qf.reshape(-1, H, K), kf.reshape(-1, H, K), vf.reshape(-1, H, vf.shape[-1])
    T = qf.shape[0]
    gf = _t(_f64(_f32(g))).reshape(T, H, K)
    bf = _t(_f64(_f32(beta))).reshape(T, H)
    al = _t(_f64(_f32(A_log))).reshape(H)
    db = _t(_f64(_f32(dt_bias))).reshape(H, K)
    cu = _offsets(cu_seqlens, T)
    N = len(cu) - 1
    S0 = (_t(_f64(initial_state)).reshape(N, H, K, vf.shape[-1]) if initial_state is not None
          else torch.zeros(N, H, K, vf.shape[-1], dtype=torch.float64))
    return qf, kf, vf, gf, bf, al, db, S0, cu


def grads_autograd(q, k, v, g, beta, A_log, dt_bias, lower_bound: float, scale: float,
                   initial_state, cu_seqlens, d_out, d_final=None):
    xs = list(_inputs(q, k, v, g, beta, A_log, dt_bias, initial_state, cu_seqlens))
    cu = xs.pop()
    for x in xs:
        x.requires_grad_(True)
    out, fin = forward_torch(*xs[:7], lower_bound, scale, xs[7], cu)
    L = (out * _t(_f64(_f32(d_out))).reshape(out.shape)).sum()
    if d_final is not None:
        L = L + (fin * _t(_f64(d_final)).reshape(fin.shape)).sum()
    gr = torch.autograd.grad(L, xs, allow_unused=True)
    return tuple(np.zeros(x.shape) if gi is None else gi.detach().numpy() for gi, x in zip(gr, xs))


def chunk_step_bwd(q, k, v, la, beta, S, scale: float, dO, dSn):
    """Backward of one chunk (single head, fp64): given the chunk's inputs, the state S
    at its start and the gradients dO (of its outputs) and dSn (of the state after it),
    returns dq, dk, dv, dla, dbeta, dS (of the state at its start) and the stages."""
    L = q.shape[0]
    G = np.cumsum(la, axis=0)
    incl = np.tril(np.ones((L, L), dtype=bool))
    strict = np.tril(np.ones((L, L), dtype=bool), -1)
    D = np.exp(np.where(incl[:, :, None], G[:, None, :] - G[None, :, :], -np.inf))
    KK = np.einsum("rc,ic,ric->ri", k, k, D)
    A = np.where(strict, beta[:, None] * KK, 0.0)
    P = np.where(incl, np.einsum("rc,ic,ric->ri", q, k, D), 0.0)
    Tm = np.linalg.inv(np.eye(L) + A)
    gam = np.exp(G)
    Xw = beta[:, None] * gam * k
    Xu = beta[:, None] * v
    W = Tm @ Xw
    U = Tm @ Xu - W @ S
    eK = np.exp(G[-1][None, :] - G)
    Khat = k * eK
    gC = np.exp(G[-1])
    # S_next = Diag(gC) S + Khat^T U
    dS = gC[:, None] * dSn
    dgC = (S * dSn).sum(axis=1)
    dKhat = U @ dSn.T
    dU = Khat @ dSn
    # O = scale ((gam q) S + P U)
    dQg = scale * dO @ S.T
    dS = dS + scale * (gam * q).T @ dO
    dP = np.where(incl, scale * dO @ U.T, 0.0)
    dU = dU + scale * P.T @ dO
    # U = T Xu - W S,  W = T Xw
    dW = -dU @ S.T
    dS = dS - W.T @ dU
    dT = dU @ Xu.T + dW @ Xw.T
    dXu = Tm.T @ dU
    dXw = Tm.T @ dW
    dA = np.where(strict, -Tm.T @ dT @ Tm.T, 0.0)
    dv = beta[:, None] * dXu
    dbeta = (dXu * v).sum(1) + (dXw * gam * k).sum(1) + (dA * KK).sum(1)
    dk = dXw * beta[:, None] * gam
    dG = dXw * beta[:, None] * gam * k
    dq = dQg * gam
    dG = dG + dQg * gam * q
    # KK_ri = sum_c k_rc k_ic D_ric (weighted by beta_r in A)
    M = (dA * beta[:, None])[:, :, None] * D
    dk = dk + np.einsum("ric,ic->rc", M, k) + np.einsum("ric,rc->ic", M, k)
    tk = M * k[:, None, :] * k[None, :, :]
    dG = dG + tk.sum(1) - tk.sum(0)
    # P_ri = sum_c q_rc k_ic D_ric
    MP = dP[:, :, None] * D
    dq = dq + np.einsum("ric,ic->rc", MP, k)
    dk = dk + np.einsum("ric,rc->ic", MP, q)
    tp = MP * q[:, None, :] * k[None, :, :]
    dG = dG + tp.sum(1) - tp.sum(0)
    # Khat = k exp(G_last - G), gC = exp(G_last)
    dk = dk + dKhat * eK
    dG = dG - dKhat * Khat
    dG[-1] += (dKhat * Khat).sum(0) + dgC * gC
    dla = np.cumsum(dG[::-1], axis=0)[::-1]
    stages = dict(Gamma=G, T=Tm, W=W, U=U, P=P, dU=dU, dA=dA, dT=dT, dG=dG)
    return dq, dk, dv, dla, dbeta, dS, stages


def gate_bwd(g, A_log, dt_bias, lower_bound: float, dla):
    """Gradients of log a = max(-exp(A_log_h) softplus(g + dt_bias_h), lower_bound) given
    dla [T, H, K]: (dg, dA_log [H], ddt_bias [H, K]); zero where the clamp is active."""
    g64 = _f64(_f32(g))
    H = g64.shape[-2]
    x = g64 + _f64(_f32(dt_bias)).reshape(H, -1)
    ea = np.exp(_f64(_f32(A_log)).reshape(H))[:, None]
    raw = -ea * np.logaddexp(0.0, x)
    free = raw >= lower_bound
    sig = 1.0 / (1.0 + np.exp(-x))
    dg = np.where(free, dla * (-ea) * sig, 0.0)
    dA_log = np.where(free, dla * raw, 0.0).sum(axis=(0, 2))
    return dg, dA_log, dg.sum(axis=0)


def grads_chunked(q, k, v, g, beta, A_log, dt_bias, lower_bound: float, scale: float,
                  initial_state, cu_seqlens, d_out, d_final=None, chunk: int = 64):
    qf, kf, vf = (bf16_to_f64(x) for x in (q, k, v))
    H, K = qf.shape[-2], qf.shape[-1]
    qf, kf, vf = qf.reshape(-1, H, K), kf.reshape(-1, H, K), vf.reshape(-1, H, vf.shape[-1])
    T, V = qf.shape[0], vf.shape[-1]
    la = gate_np(_f32(g).reshape(T, H, K), A_log, dt_bias, lower_bound)
    bt = _f64(_f32(beta)).reshape(T, H)
    dO = _f64(_f32(d_out)).reshape(T, H, V)
    cu = _offsets(cu_seqlens, T)
    N = len(cu) - 1
    S0 = (_f64(initial_state).reshape(N, H, K, V) if initial_state is not None else np.zeros((N, H, K, V)))
    dq, dk, dv, dla = (np.zeros((T, H, K)), np.zeros((T, H, K)), np.zeros((T, H, V)), np.zeros((T, H, K)))
    dbeta, dS0 = np.zeros((T, H)), np.zeros((N, H, K, V))
    for n in range(N):
        b0, b1 = int(cu[n]), int(cu[n + 1])
        starts = list(range(b0, b1, chunk))
        for h in range(H):
            S, states = S0[n, h].copy(), []
            for t0 in starts:                       # forward: chunk-start states
                states.append(S.copy())
                t1 = min(t0 + chunk, b1)
                G = np.cumsum(la[t0:t1, h], axis=0)
                # the chunk's state update, as in the forward
                from . import chunk_step
                _, S, _ = chunk_step(qf[t0:t1, h], kf[t0:t1, h], vf[t0:t1, h], la[t0:t1, h],
                                     bt[t0:t1, h], S, scale)
            dSn = (_f64(d_final).reshape(N, H, K, V)[n, h].copy() if d_final is not None
                   else np.zeros((K, V)))
            for ci in range(len(starts) - 1, -1, -1):
                t0 = starts[ci]
                t1 = min(t0 + chunk, b1)
                r = chunk_step_bwd(qf[t0:t1, h], kf[t0:t1, h], vf[t0:t1, h], la[t0:t1, h], bt[t0:t1, h],
                                   states[ci], scale, dO[t0:t1, h], dSn)
                dq[t0:t1, h], dk[t0:t1, h], dv[t0:t1, h], dla[t0:t1, h], dbeta[t0:t1, h], dSn = r[:6]
            dS0[n, h] = dSn
    dg, dA_log, ddt = gate_bwd(g, A_log, dt_bias, lower_bound, dla.reshape(T, H, K))
    return dq, dk, dv, dg, dbeta, dA_log, ddt, dS0
