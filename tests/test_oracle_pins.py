"""Pins of the fp64 oracle to things other than itself (CPU only).

Each test checks the oracle against a closed form, a library routine, an
independently derived formulation (DeltaNet / Gated DeltaNet chunked forms,
brute-force linear attention) or an invariant of the recurrence.  Together
they catch a dropped term, a wrong sign, the wrong decay side or order, a
missing scale, a wrong gate, or a mis-indexed varlen offset.
"""
import math
import os

import numpy as np
import pytest
import torch

import kda_workloads as W
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(x):
    return torch.as_tensor(np.asarray(x), dtype=torch.float32).to(torch.bfloat16)


def _rand_unit_keys(rng, T, H, K, nnz=4):
    """Keys with exactly unit norm in bf16: nnz entries of +-0.5 (nnz = 4)."""
    k = np.zeros((T, H, K), np.float32)
    for t in range(T):
        for h in range(H):
            idx = rng.choice(K, size=nnz, replace=False)
            k[t, h, idx] = rng.choice([-0.5, 0.5], size=nnz)
    return k


# ----------------------------------------------------------------------------
# input widening and the gate

def test_bf16_widening_is_exact():
    bits = np.arange(65536, dtype=np.uint16)
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    ref = t.double().numpy()                         # torch's own widening
    got = oracle.bf16_to_f64(bits)
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.all(np.isnan(got[~finite]) == np.isnan(ref[~finite]))


def test_gate_golden_points():
    rows = []
    with open(os.path.join(GOLDEN, "gate_points.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append([float(x) for x in line.split()])
    for g, dtb, alog, lb, expect, tol in rows:
        la = oracle.gate(np.full((1, 1, 1), g, np.float32), np.array([alog], np.float32),
                         np.full((1, 1), dtb, np.float32), lb)[0, 0, 0]
        assert abs(la - expect) <= tol, (g, dtb, alog, lb, la, expect)


def test_gate_matches_library_softplus_and_clamp():
    rng = np.random.default_rng(5)
    g = rng.normal(0, 3, size=(64, 3, 128)).astype(np.float32)
    A_log = np.log(rng.uniform(1, 16, size=3)).astype(np.float32)
    dtb = rng.normal(0, 0.1, size=(3, 128)).astype(np.float32)
    for lb in (-5.0, -float("inf")):
        la = oracle.gate(g, A_log, dtb, lb)
        x = g.astype(np.float64) + dtb[None].astype(np.float64)
        sp = np.logaddexp(0.0, x)                         # library softplus
        raw = -np.exp(A_log.astype(np.float64))[None, :, None] * sp
        assert np.all(la <= 0.0) and np.all(la >= lb)
        np.testing.assert_allclose(la, np.maximum(raw, lb), rtol=1e-14, atol=1e-300)
        # the numpy gate of the chunked form agrees with the C gate
        np.testing.assert_allclose(oracle.gate_np(g, A_log, dtb, lb), la, rtol=1e-14, atol=1e-300)


# ----------------------------------------------------------------------------
# closed forms of the recurrence

def _decay_pattern_inputs(T, H, K, V, rng):
    """Gate inputs whose decays are known in closed form per channel:
    channel c % 3 == 0: x = 0 -> log a = -ln 2; c % 3 == 1: x = -40 -> a = 1 (to
    double precision); c % 3 == 2: x = 40 -> clamped at lb = -5."""
    dtb = np.zeros((H, K), np.float32)
    dtb[:, 1::3] = -40.0
    dtb[:, 2::3] = 40.0
    g = np.zeros((T, H, K), np.float32)
    A_log = np.zeros(H, np.float32)
    per_token = np.zeros(K)
    per_token[0::3] = -math.log(2.0)
    per_token[1::3] = -math.log1p(math.exp(-40.0))
    per_token[2::3] = -5.0
    return g, A_log, dtb, per_token


def test_beta_zero_is_pure_decay():
    rng = np.random.default_rng(0)
    T, H, K, V = 37, 2, 128, 128
    g, A_log, dtb, per_token = _decay_pattern_inputs(T, H, K, V, rng)
    q = _bf16(rng.normal(size=(T, H, K)))
    k = _bf16(rng.normal(size=(T, H, K)))
    v = _bf16(rng.normal(size=(T, H, V)))
    beta = np.zeros((T, H), np.float32)
    S0 = rng.normal(size=(1, H, K, V))
    scale = 0.37
    out, fin = oracle.recurrent(q, k, v, g, beta, A_log, dtb, -5.0, scale, S0)
    qf = q.double().numpy()
    for t in range(T):
        d = np.exp((t + 1) * per_token)                  # Diag(e^{sum la}) acts on rows
        St = d[None, :, None] * S0[0]
        expect = scale * np.einsum("hkv,hk->hv", St, qf[t])
        np.testing.assert_allclose(out[t], expect, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(fin[0], np.exp(T * per_token)[None, :, None] * S0[0],
                               rtol=1e-12, atol=1e-300)


def test_one_hot_delta_write_replaces_a_row():
    rng = np.random.default_rng(1)
    T, H, K, V = 12, 1, 128, 128
    js = rng.choice(K, size=T)
    k = np.zeros((T, H, K), np.float32)
    k[np.arange(T), 0, js] = 1.0
    v = _bf16(rng.normal(size=(T, H, V)))
    q = _bf16(rng.normal(size=(T, H, K)))
    g = np.full((T, H, K), -40.0, np.float32)          # a = 1 to double precision
    beta = np.ones((T, H), np.float32)
    S0 = rng.normal(size=(1, H, K, V))
    expect = S0[0, 0].copy()
    vf = v.double().numpy()
    for t in range(1, T + 1):
        _, fin = oracle.recurrent(q[:t], _bf16(k[:t]), v[:t], g[:t], beta[:t],
                                  np.zeros(1, np.float32), np.zeros((1, K), np.float32),
                                  -5.0, 1.0, S0)
        expect[js[t - 1]] = vf[t - 1, 0]
        np.testing.assert_allclose(fin[0, 0], expect, rtol=1e-15, atol=1e-15)


def test_unit_key_query_reads_back_value():
    # beta = 1, q_t = k_t, |k_t| = 1  =>  o_t = scale * v_t whatever the history and gates.
    rng = np.random.default_rng(2)
    T, H, K, V = 40, 2, 128, 128
    k = _bf16(_rand_unit_keys(rng, T, H, K))
    v = _bf16(rng.normal(size=(T, H, V)))
    g = rng.normal(size=(T, H, K)).astype(np.float32)
    beta = np.ones((T, H), np.float32)
    A_log = np.log(rng.uniform(1, 16, size=H)).astype(np.float32)
    dtb = rng.normal(0, 0.1, size=(H, K)).astype(np.float32)
    S0 = rng.normal(size=(1, H, K, V))
    scale = 0.125
    out, _ = oracle.recurrent(k, k, v, g, beta, A_log, dtb, -5.0, scale, S0)
    np.testing.assert_allclose(out, scale * v.double().numpy(), rtol=0, atol=1e-13)


# ----------------------------------------------------------------------------
# special cases that reduce to known recurrences, each in its own chunked form

def _deltanet_chunked(q, k, v, beta, S, scale, C=16):
    """DeltaNet (a = 1) in the WY chunked form, matrices only, no decays."""
    T = q.shape[0]
    out = np.zeros_like(v)
    for t0 in range(0, T, C):
        Q, Kc, Vc, b = q[t0:t0 + C], k[t0:t0 + C], v[t0:t0 + C], beta[t0:t0 + C]
        L = Q.shape[0]
        A = np.tril(b[:, None] * (Kc @ Kc.T), -1)
        Tm = np.linalg.inv(np.eye(L) + A)
        Wm = Tm @ (b[:, None] * Kc)
        U = Tm @ (b[:, None] * Vc) - Wm @ S
        out[t0:t0 + C] = scale * (Q @ S + np.tril(Q @ Kc.T) @ U)
        S = S + Kc.T @ U
    return out, S


def _gdn_chunked(q, k, v, beta, la, S, scale, C=16):
    """Gated DeltaNet (one scalar decay per token) in chunked form: the decay
    factors exp(G_r - G_i) form a scalar mask on plain matmuls."""
    T = q.shape[0]
    out = np.zeros_like(v)
    for t0 in range(0, T, C):
        Q, Kc, Vc, b, l = q[t0:t0 + C], k[t0:t0 + C], v[t0:t0 + C], beta[t0:t0 + C], la[t0:t0 + C]
        L = Q.shape[0]
        G = np.cumsum(l)
        M = np.exp(np.where(np.tril(np.ones((L, L), bool)), G[:, None] - G[None, :], -np.inf))
        A = np.tril(b[:, None] * (Kc @ Kc.T) * M, -1)
        Tm = np.linalg.inv(np.eye(L) + A)
        Wm = Tm @ (b[:, None] * np.exp(G)[:, None] * Kc)
        U = Tm @ (b[:, None] * Vc) - Wm @ S
        out[t0:t0 + C] = scale * (np.exp(G)[:, None] * Q @ S + (Q @ Kc.T * M) @ U)
        S = np.exp(G[-1]) * S + (np.exp(G[-1] - G)[:, None] * Kc).T @ U
    return out, S


def _small_case(rng, T=50, H=2, K=128, V=128):
    q = _bf16(rng.normal(size=(T, H, K)) / math.sqrt(K))
    k = _bf16(rng.normal(size=(T, H, K)) / math.sqrt(K))
    v = _bf16(rng.normal(size=(T, H, V)))
    beta = (1 / (1 + np.exp(-rng.normal(size=(T, H))))).astype(np.float32)
    S0 = rng.normal(0, 0.1, size=(1, H, K, V))
    return q, k, v, beta, S0


def test_alpha_one_is_deltanet():
    rng = np.random.default_rng(3)
    q, k, v, beta, S0 = _small_case(rng)
    T, H, K = q.shape
    la = np.zeros((T, H, K), np.float32)
    out, fin = oracle.recurrent(q, k, v, la, beta, None, None, -5.0, 0.3, S0, gate_mode=1)
    qf, kf, vf = (x.double().numpy() for x in (q, k, v))
    for h in range(H):
        o_ref, s_ref = _deltanet_chunked(qf[:, h], kf[:, h], vf[:, h], beta[:, h].astype(np.float64),
                                         S0[0, h], 0.3)
        np.testing.assert_allclose(out[:, h], o_ref, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(fin[0, h], s_ref, rtol=1e-10, atol=1e-12)


def test_channel_uniform_alpha_is_gated_deltanet():
    rng = np.random.default_rng(4)
    q, k, v, beta, S0 = _small_case(rng)
    T, H, K = q.shape
    la_tok = -rng.uniform(0.0, 2.0, size=(T, H))
    la = np.repeat(la_tok[:, :, None], K, axis=2).astype(np.float32)
    out, fin = oracle.recurrent(q, k, v, la, beta, None, None, -5.0, 0.7, S0, gate_mode=1)
    qf, kf, vf = (x.double().numpy() for x in (q, k, v))
    for h in range(H):
        o_ref, s_ref = _gdn_chunked(qf[:, h], kf[:, h], vf[:, h], beta[:, h].astype(np.float64),
                                    la[:, h, 0].astype(np.float64), S0[0, h], 0.7)
        np.testing.assert_allclose(out[:, h], o_ref, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(fin[0, h], s_ref, rtol=1e-10, atol=1e-12)


def test_gdn_wrapper_is_scalar_decay_chunked_form():
    """gdn_recurrent (one gate input per token-head, dt_bias per head) equals the
    independent chunked Gated DeltaNet form with the gate evaluated token by token."""
    rng = np.random.default_rng(11)
    q, k, v, beta, S0 = _small_case(rng, T=45)
    T, H, K = q.shape
    g = rng.normal(size=(T, H)).astype(np.float32)
    A_log = np.log(rng.uniform(1, 16, size=H)).astype(np.float32)
    dt_bias = (0.1 * rng.normal(size=H)).astype(np.float32)
    out, fin = oracle.gdn_recurrent(q, k, v, g, beta, A_log, dt_bias, -4.0, 0.5, S0)
    la = oracle.gate_np(g[:, :, None], A_log, dt_bias[:, None], -4.0)[:, :, 0]
    qf, kf, vf = (x.double().numpy() for x in (q, k, v))
    for h in range(H):
        o_ref, s_ref = _gdn_chunked(qf[:, h], kf[:, h], vf[:, h], beta[:, h].astype(np.float64),
                                    la[:, h], S0[0, h], 0.5)
        np.testing.assert_allclose(out[:, h], o_ref, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(fin[0, h], s_ref, rtol=1e-10, atol=1e-12)


def test_additive_update_is_linear_attention():
    rng = np.random.default_rng(6)
    q, k, v, beta, S0 = _small_case(rng, T=33)
    T, H, K = q.shape
    qf, kf, vf = (x.double().numpy() for x in (q, k, v))
    # a = 1: o_t = scale (S0^T q_t + sum_{i<=t} beta_i (q_t . k_i) v_i)
    la = np.zeros((T, H, K), np.float32)
    out, _ = oracle.recurrent(q, k, v, la, beta, None, None, -5.0, 0.5, S0,
                              gate_mode=1, additive=True)
    for h in range(H):
        ref = 0.5 * (qf[:, h] @ S0[0, h] + np.tril(qf[:, h] @ kf[:, h].T) @ (beta[:, h, None] * vf[:, h]))
        np.testing.assert_allclose(out[:, h], ref, rtol=1e-12, atol=1e-14)
    # channel-wise decay: o_t = scale (sum_c q_tc e^{G_tc} S0[c] + sum_{i<=t} beta_i sum_c q_tc k_ic e^{G_tc - G_ic} v_i)
    la = (-rng.uniform(0, 1.5, size=(T, H, K))).astype(np.float32)
    out, _ = oracle.recurrent(q, k, v, la, beta, None, None, -5.0, 0.5, S0,
                              gate_mode=1, additive=True)
    for h in range(H):
        G = np.cumsum(la[:, h].astype(np.float64), axis=0)
        ref = np.zeros((T, v.shape[-1]))
        for t in range(T):
            ref[t] = (qf[t, h] * np.exp(G[t])) @ S0[0, h]
            for i in range(t + 1):
                ref[t] += beta[i, h] * np.sum(qf[t, h] * kf[i, h] * np.exp(G[t] - G[i])) * vf[i, h]
        np.testing.assert_allclose(out[:, h], 0.5 * ref, rtol=1e-11, atol=1e-14)


# ----------------------------------------------------------------------------
# structural invariants

def _call(x, **kw):
    return oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"],
                            x["lower_bound"], x["scale"], x["initial_state"], x["cu_seqlens"], **kw)


def test_varlen_equals_independent_sequences():
    w = W.custom([70, 0, 129, 64, 5], H=3, init="normal")
    x = W.make_inputs(w)
    out, fin = _call(x)
    cu = x["cu_seqlens"].tolist()
    for n in range(w.N):
        a, b = cu[n], cu[n + 1]
        sub = dict(x)
        for key in ("q", "k", "v", "g", "beta"):
            sub[key] = x[key][a:b]
        sub["initial_state"] = x["initial_state"][n:n + 1]
        sub["cu_seqlens"] = None
        o_n, f_n = _call(sub)
        np.testing.assert_array_equal(out[a:b], o_n)
        np.testing.assert_array_equal(fin[n], f_n[0])
    # an empty sequence passes its initial state through
    np.testing.assert_array_equal(fin[1], x["initial_state"][1].double().numpy())


def test_split_and_resume_equals_full_run():
    w = W.custom([300], H=2, packed=False, init="normal")
    x = W.make_inputs(w)
    out, fin = _call(x)
    for t1 in (1, 64, 150, 299):
        a = dict(x)
        b = dict(x)
        for key in ("q", "k", "v", "g", "beta"):
            a[key] = x[key][:t1]
            b[key] = x[key][t1:]
        oa, fa = _call(a)
        b["initial_state"] = torch.from_numpy(fa)
        ob, fb = _call(b)
        np.testing.assert_allclose(np.concatenate([oa, ob]), out, rtol=0, atol=1e-15)
        np.testing.assert_allclose(fb, fin, rtol=0, atol=1e-15)


@pytest.mark.parametrize("seq_lens,lb,init", [
    ((256,), -5.0, "zero"),
    ((200, 77, 0, 130), -5.0, "normal"),
    ((65, 63, 1), -20.0, "normal"),
    ((150,), -float("inf"), None),
])
def test_chunked_equals_recurrent(seq_lens, lb, init):
    w = W.custom(seq_lens, H=2, init=init, lower_bound=lb)
    x = W.make_inputs(w)
    o_r, f_r = _call(x)
    o_c, f_c = oracle.chunked(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"],
                              x["lower_bound"], x["scale"], x["initial_state"], x["cu_seqlens"])
    assert oracle.rel_l2(o_c, o_r) <= 1e-10
    assert oracle.rel_l2(f_c, f_r) <= 1e-10


def test_state_norm_contraction():
    # |k| = 1, beta in [0,1], a <= 1  =>  |S_t|_2 <= |S_{t-1}|_2 + beta_t |v_t|_2
    rng = np.random.default_rng(8)
    T, H, K, V = 24, 1, 128, 128
    k = _bf16(_rand_unit_keys(rng, T, H, K))
    q = _bf16(rng.normal(size=(T, H, K)))
    v = _bf16(rng.normal(size=(T, H, V)))
    g = rng.normal(size=(T, H, K)).astype(np.float32)
    beta = rng.uniform(0, 1, size=(T, H)).astype(np.float32)
    A_log = np.zeros(H, np.float32)
    dtb = np.zeros((H, K), np.float32)
    S0 = rng.normal(size=(1, H, K, V))
    prev = np.linalg.norm(S0[0, 0], 2)
    vf = v.double().numpy()
    for t in range(1, T + 1):
        _, fin = oracle.recurrent(q[:t], k[:t], v[:t], g[:t], beta[:t], A_log, dtb, -5.0, 1.0, S0)
        cur = np.linalg.norm(fin[0, 0], 2)
        assert cur <= prev + beta[t - 1, 0] * np.linalg.norm(vf[t - 1, 0]) + 1e-12
        prev = cur


def test_linear_in_values_and_initial_state():
    rng = np.random.default_rng(9)
    T, H, K, V = 45, 2, 128, 128
    x = W.make_inputs(W.custom([T], H=H, packed=False, init="normal"))
    v1 = rng.integers(-8, 9, size=(T, H, V)) / 8.0          # sums stay exact in bf16
    v2 = rng.integers(-8, 9, size=(T, H, V)) / 8.0
    s1 = rng.normal(size=(1, H, K, V))
    s2 = rng.normal(size=(1, H, K, V))

    def run(vv, ss):
        y = dict(x)
        y["v"] = _bf16(vv)
        y["initial_state"] = torch.from_numpy(ss)
        return _call(y)

    o1, f1 = run(v1, s1)
    o2, f2 = run(v2, s2)
    o3, f3 = run(v1 + v2, s1 + s2)
    np.testing.assert_allclose(o3, o1 + o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(f3, f1 + f2, rtol=1e-12, atol=1e-13)


def test_null_initial_state_equals_explicit_zeros():
    x = W.make_inputs(W.custom([100, 30], H=2, init="zero"))
    o_z, f_z = _call(x)
    y = dict(x)
    y["initial_state"] = None
    o_n, f_n = _call(y)
    np.testing.assert_array_equal(o_z, o_n)
    np.testing.assert_array_equal(f_z, f_n)
