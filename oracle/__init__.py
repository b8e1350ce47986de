"""fp64 CPU oracle for the KDA chunked-prefill forward.

TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and the CPU-baseline
leg of bench.py may import this package.  It shares no code with the CUDA
library (gated_delta_rule_135_b200) and never imports it.

Two independent formulations of the same map:

* ``recurrent``: the token-by-token definition in C (kda_ref.c), fp64,
  OpenMP over (sequence, head) pairs.  This is the reference every GPU result
  is compared with.
* ``chunked``: the chunked (WY / UT-transform) form in numpy fp64, written
  from the algebra of the recurrence, computing every intra-chunk decay
  exp(Gamma_r - Gamma_i) directly.  It agrees with ``recurrent`` to ~1e-15 and
  also returns its per-stage intermediates (Gamma, A, T, W, U~, U, P, chunk
  states) so GPU stages can be checked one at a time.

Method source: FlashKDA posts (donniechu.com, section "Số liệu kỹ thuật";
toolarium.ru, section "Где ограничения прямо сейчас"): KDA is a gated delta
rule with fine-grained channel-wise decay, K = V = 128, bf16 + fp32, varlen
via cu_seqlens, initial/final states, gate parameters A_log, dt_bias,
lower_bound.  The pages print no formula; the gate and recurrence used here
are the library's specification, restated in kda_ref.c.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        c_p = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.kda_oracle_recurrent.restype = ctypes.c_int
        lib.kda_oracle_recurrent.argtypes = [
            c_p, c_p, c_p, c_p, c_p, c_p, c_p,
            ctypes.c_double, ctypes.c_double,
            c_p, c_p,
            i64, i64, i64, i64, i64,
            ctypes.c_int, ctypes.c_int,
            c_p, c_p, ctypes.c_int]
        lib.kda_oracle_gate.restype = None
        lib.kda_oracle_gate.argtypes = [c_p, c_p, c_p, ctypes.c_double,
                                        i64, i64, i64, c_p]
        lib.kda_oracle_bf16_to_f64.restype = None
        lib.kda_oracle_bf16_to_f64.argtypes = [c_p, c_p, i64]
        lib.kda_oracle_max_threads.restype = ctypes.c_int
        lib.kda_oracle_max_threads.argtypes = []
        _lib = lib
    return _lib


# ----------------------------------------------------------------------------
# array plumbing (torch CPU tensors or numpy arrays in; numpy out)

def _bf16_bits(x) -> np.ndarray:
    """Raw bf16 bit patterns (uint16) of a bf16 torch tensor, or pass-through
    for a uint16 numpy array."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    assert x.dtype == torch.bfloat16, x.dtype
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _f32(x) -> np.ndarray:
    if isinstance(x, np.ndarray):
        return np.ascontiguousarray(x, dtype=np.float32)
    return np.ascontiguousarray(x.detach().cpu().float().numpy())


def _f64(x) -> np.ndarray:
    if isinstance(x, np.ndarray):
        return np.ascontiguousarray(x, dtype=np.float64)
    return np.ascontiguousarray(x.detach().cpu().double().numpy())


def bf16_to_f64(x) -> np.ndarray:
    """Exact widening of bf16 values to float64 (done by the oracle's C code)."""
    bits = _bf16_bits(x)
    out = np.empty(bits.shape, dtype=np.float64)
    _load().kda_oracle_bf16_to_f64(bits.ctypes.data, out.ctypes.data, bits.size)
    return out


def max_threads() -> int:
    return int(_load().kda_oracle_max_threads())


def _offsets(cu_seqlens, T: int) -> np.ndarray:
    if cu_seqlens is None:
        return np.array([0, T], dtype=np.int64)
    if isinstance(cu_seqlens, np.ndarray):
        cu = cu_seqlens.astype(np.int64)
    else:
        cu = cu_seqlens.detach().cpu().numpy().astype(np.int64)
    return np.ascontiguousarray(cu)


def fixed_offsets(batch: int, seqlen: int) -> np.ndarray:
    """cu_seqlens equivalent of a [batch, seqlen] fixed-length layout."""
    return np.arange(batch + 1, dtype=np.int64) * seqlen


# ----------------------------------------------------------------------------
# the gate

def gate(g, A_log, dt_bias, lower_bound: float) -> np.ndarray:
    """log a = max(-exp(A_log_h) * softplus(g + dt_bias_h), lower_bound), fp64.

    g: [T, H, K] float32; A_log: [H]; dt_bias: [H, K].  Returns [T, H, K] float64.
    """
    g32 = _f32(g)
    T, H, K = g32.shape
    la = np.empty(g32.shape, dtype=np.float64)
    _load().kda_oracle_gate(g32.ctypes.data, _f32(A_log).ctypes.data,
                            _f32(dt_bias).ctypes.data, float(lower_bound),
                            T, H, K, la.ctypes.data)
    return la


# ----------------------------------------------------------------------------
# the recurrence (reference)

def recurrent(q, k, v, g, beta, A_log, dt_bias, lower_bound: float, scale: float,
              initial_state=None, cu_seqlens=None, *, gate_mode: int = 0,
              additive: bool = False, nthreads: int = 0, want_final: bool = True):
    """Token-by-token fp64 KDA forward.

    q, k: [T, H, K] bf16; v: [T, H, V] bf16; g: [T, H, K] float32 (gate_mode=1:
    g already holds log a and the gate is bypassed); beta: [T, H] float32;
    A_log: [H]; dt_bias: [H, K]; initial_state: [N, H, K, V] or None;
    cu_seqlens: [N + 1] offsets or None (one sequence of length T).
    Leading batch dims of q/k/v/g/beta are flattened into T (the packed layout).
    Returns (out [T, H, V] float64, final_state [N, H, K, V] float64 or None).
    """
    qb = _bf16_bits(q)
    kb = _bf16_bits(k)
    vb = _bf16_bits(v)
    K = qb.shape[-1]
    V = vb.shape[-1]
    H = qb.shape[-2]
    qb = qb.reshape(-1, H, K)
    kb = kb.reshape(-1, H, K)
    vb = vb.reshape(-1, H, V)
    T = qb.shape[0]
    g32 = _f32(g).reshape(T, H, K)
    b32 = _f32(beta).reshape(T, H)
    a32 = _f32(A_log).reshape(H) if A_log is not None else np.zeros(H, np.float32)
    d32 = _f32(dt_bias).reshape(H, K) if dt_bias is not None else np.zeros((H, K), np.float32)
    cu = _offsets(cu_seqlens, T)
    N = cu.shape[0] - 1
    assert cu[0] == 0 and cu[-1] == T and np.all(np.diff(cu) >= 0)
    s0 = None
    if initial_state is not None:
        s0 = _f64(initial_state).reshape(N, H, K, V)
    out = np.empty((T, H, V), dtype=np.float64)
    fin = np.empty((N, H, K, V), dtype=np.float64) if want_final else None
    rc = _load().kda_oracle_recurrent(
        qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, g32.ctypes.data,
        b32.ctypes.data, a32.ctypes.data, d32.ctypes.data,
        float(lower_bound), float(scale),
        s0.ctypes.data if s0 is not None else None, cu.ctypes.data,
        N, T, H, K, V, int(gate_mode), int(bool(additive)),
        out.ctypes.data, fin.ctypes.data if fin is not None else None, int(nthreads))
    if rc != 0:
        raise MemoryError("oracle: allocation failed")
    return out, fin


# ----------------------------------------------------------------------------
# the chunked form (second, independent formulation)

def gdn_recurrent(q, k, v, g, beta, A_log, dt_bias, lower_bound: float, scale: float,
                  initial_state=None, cu_seqlens=None, **kw):
    """Scalar-gate variant (Gated DeltaNet): the recurrence above with one decay per
    (token, head), log a_t = max(-exp(A_log_h) softplus(g_t,h + dt_bias_h), lower_bound),
    shared by all K channels.  g: [T, H] (or leading batch dims); dt_bias: [H].  It is
    ``recurrent`` with g and dt_bias repeated over the channel axis.  The FlashKDA H20
    table (toolarium.ru, section "Что показывают H20-бенчмарки") compares against
    such a "gdn" kernel.
    """
    g32 = _f32(g)
    H = g32.shape[-1]
    K = (q.shape[-1] if hasattr(q, "shape") else 128)
    g3 = np.repeat(g32.reshape(-1, H)[:, :, None], K, axis=2)
    db = np.repeat(_f32(dt_bias).reshape(H, 1), K, axis=1)
    return recurrent(q, k, v, g3, beta, A_log, db, lower_bound, scale, initial_state,
                     cu_seqlens, **kw)


def _softplus_np(x: np.ndarray) -> np.ndarray:
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def gate_np(g, A_log, dt_bias, lower_bound: float) -> np.ndarray:
    """The same gate written in numpy (used by the chunked form)."""
    g64 = _f64(g)
    H = g64.shape[-2]
    a = np.exp(_f64(A_log).reshape(H))[:, None]
    d = _f64(dt_bias).reshape(H, -1)
    la = -a * _softplus_np(g64 + d)
    return np.maximum(la, lower_bound)


def chunk_step(q, k, v, la, beta, S, scale: float):
    """One chunk of the chunked form for a single head, all fp64.

    q, k: [L, K]; v: [L, V]; la: [L, K] log-decay; beta: [L]; S: [K, V] state
    at the chunk start.  Returns (o [L, V], S_next [K, V], stages dict).

    Within the chunk, with Gamma_r = sum_{i<=r} la_i (inclusive) and
    gamma_r = exp(Gamma_r):
      S_r = Diag(gamma_r) S_0 + sum_{i<=r} Diag(gamma_r / gamma_i) k_i u_i^T,
      u_r = beta_r (v_r - S_{r-1}^T (a_r * k_r)),
    which gives (I + A) U = diag(beta) (V - (gamma*K) S_0) with
      A_ri = beta_r sum_c k_rc k_ic gamma_rc / gamma_ic  (i < r), so
      U = T diag(beta) V - T diag(beta) (gamma*K) S_0 = U~ - W S_0,
      O = scale ((gamma*Q) S_0 + P U),  P_ri = sum_c q_rc k_ic gamma_rc/gamma_ic (i <= r),
      S_L = Diag(gamma_L) S_0 + Khat^T U,  Khat_i = k_i * gamma_L / gamma_i.
    """
    L = q.shape[0]
    G = np.cumsum(la, axis=0)                           # [L, K]
    diff = G[:, None, :] - G[None, :, :]                # [r, i, K] = Gamma_r - Gamma_i
    incl = np.tril(np.ones((L, L), dtype=bool))         # i <= r
    strict = np.tril(np.ones((L, L), dtype=bool), -1)   # i <  r
    D = np.exp(np.where(incl[:, :, None], diff, -np.inf))  # 0 above the diagonal
    KK = np.einsum("rc,ic,ric->ri", k, k, D)
    A = np.where(strict, beta[:, None] * KK, 0.0)
    P = np.where(incl, np.einsum("rc,ic,ric->ri", q, k, D), 0.0)
    Tm = np.linalg.inv(np.eye(L) + A)
    gam = np.exp(G)
    W = Tm @ (beta[:, None] * gam * k)
    Ut = Tm @ (beta[:, None] * v)
    U = Ut - W @ S
    o = scale * ((gam * q) @ S + P @ U)
    Khat = k * np.exp(G[-1][None, :] - G)
    S_next = np.exp(G[-1])[:, None] * S + Khat.T @ U
    stages = dict(Gamma=G, A=A, T=Tm, W=W, Ut=Ut, U=U, P=P, S0=S.copy())
    return o, S_next, stages


def chunked(q, k, v, g, beta, A_log, dt_bias, lower_bound: float, scale: float,
            initial_state=None, cu_seqlens=None, *, chunk: int = 64,
            gate_mode: int = 0, keep_stages: bool = False):
    """Chunked fp64 KDA forward (chunks restart at every sequence start).

    Same arguments and results as ``recurrent``; with keep_stages=True also
    returns a list, per (n, h), of per-chunk stage dicts.
    """
    qf = bf16_to_f64(q)
    kf = bf16_to_f64(k)
    vf = bf16_to_f64(v)
    H, K = qf.shape[-2], qf.shape[-1]
    V = vf.shape[-1]
    qf = qf.reshape(-1, H, K)
    kf = kf.reshape(-1, H, K)
    vf = vf.reshape(-1, H, V)
    T = qf.shape[0]
    if gate_mode == 0:
        la = gate_np(_f32(g).reshape(T, H, K), A_log, dt_bias, lower_bound)
    else:
        la = _f64(_f32(g)).reshape(T, H, K)
    bt = _f64(_f32(beta)).reshape(T, H)
    cu = _offsets(cu_seqlens, T)
    N = cu.shape[0] - 1
    out = np.zeros((T, H, V))
    fin = np.zeros((N, H, K, V))
    all_stages = {}
    for n in range(N):
        for h in range(H):
            S = (_f64(initial_state).reshape(N, H, K, V)[n, h].copy()
                 if initial_state is not None else np.zeros((K, V)))
            st_list = []
            for t0 in range(int(cu[n]), int(cu[n + 1]), chunk):
                t1 = min(t0 + chunk, int(cu[n + 1]))
                o, S, st = chunk_step(qf[t0:t1, h], kf[t0:t1, h], vf[t0:t1, h],
                                      la[t0:t1, h], bt[t0:t1, h], S, scale)
                out[t0:t1, h] = o
                if keep_stages:
                    st["t0"] = t0
                    st_list.append(st)
            fin[n, h] = S
            if keep_stages:
                all_stages[(n, h)] = st_list
    if keep_stages:
        return out, fin, all_stages
    return out, fin


# ----------------------------------------------------------------------------
# error measures used by the parity tests

def rel_l2(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    if den == 0.0:
        return float(num)
    return float(num / den)


def max_abs(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if x.size == 0:
        return 0.0
    return float(np.max(np.abs(x - ref)))
