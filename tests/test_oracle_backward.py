"""Pins of the backward oracle (oracle/backward.py): its torch forward equals the C
oracle, its autograd gradients equal central finite differences, and the hand-derived
chunked backward equals autograd."""
import numpy as np
import pytest
import torch

import kda_workloads as W
import oracle
from oracle import backward as B


def _case(seq_lens, H=2, lb=-5.0, packed=True, wid=81):
    w = W.custom(seq_lens, H=H, packed=packed, init="normal", lower_bound=lb, wid=wid)
    x = W.make_inputs(w)
    gen = torch.Generator().manual_seed(wid)
    dO = torch.randn(w.T, H, 128, generator=gen)
    dF = torch.randn(w.N, H, 128, 128, generator=gen) * 0.1
    return x, dO, dF


def _args(x, dO):
    return (x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"], x["lower_bound"], x["scale"],
            x["initial_state"], x["cu_seqlens"], dO)


def test_torch_forward_equals_c_oracle():
    x, _, _ = _case([70, 45])
    xs = B._inputs(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"], x["initial_state"],
                   x["cu_seqlens"])
    out, fin = B.forward_torch(*xs[:7], x["lower_bound"], x["scale"], xs[7], xs[8])
    ro, rf = oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"],
                              x["lower_bound"], x["scale"], x["initial_state"], x["cu_seqlens"])
    assert oracle.rel_l2(out.numpy(), ro) < 1e-13
    assert oracle.rel_l2(fin.numpy(), rf) < 1e-13


def test_autograd_equals_finite_differences():
    """<grad, d> against (L(x + eps d) - L(x - eps d)) / (2 eps) for every input, fp64."""
    rng = np.random.default_rng(9)
    T, H, K = 9, 2, 128
    mk = lambda *s, sc=1.0: torch.tensor(rng.normal(size=s) * sc)   # noqa: E731
    q, k = mk(T, H, K, sc=0.09), mk(T, H, K, sc=0.09)
    v, g = mk(T, H, K), mk(T, H, K)
    beta = torch.sigmoid(mk(T, H))
    A_log, dt_bias = torch.log(torch.tensor(rng.uniform(1, 4, size=H))), mk(H, K, sc=0.1)
    S0 = mk(1, H, K, K, sc=0.05)
    dO, dF = mk(T, H, K), mk(1, H, K, K, sc=0.1)
    cu = np.array([0, T])
    lb = -30.0   # the clamp stays inactive, where the map is smooth

    def loss(xs):
        out, fin = B.forward_torch(*xs[:7], lb, 0.3, xs[7], cu)
        return (out * dO).sum() + (fin * dF).sum()

    xs = [q, k, v, g, beta, A_log, dt_bias, S0]
    xs_req = [x.clone().requires_grad_(True) for x in xs]
    grads = torch.autograd.grad(loss(xs_req), xs_req)
    eps = 1e-6
    for i, (x, gr) in enumerate(zip(xs, grads)):
        d = torch.tensor(rng.normal(size=tuple(x.shape)))
        plus = [y.clone() for y in xs]
        minus = [y.clone() for y in xs]
        plus[i] = x + eps * d
        minus[i] = x - eps * d
        fd = (loss(plus) - loss(minus)).item() / (2 * eps)
        an = (gr * d).sum().item()
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (i, fd, an)


@pytest.mark.parametrize("seq_lens,lb,packed", [([70, 45], -5.0, True), ([130], -0.7, False),
                                                ([64, 1, 100], -20.0, True)],
                         ids=["varlen", "mild_gate_clamped_often", "steep_ragged"])
def test_chunked_backward_equals_autograd(seq_lens, lb, packed):
    x, dO, dF = _case(seq_lens, lb=lb, packed=packed)
    ga = B.grads_autograd(*_args(x, dO), dF)
    gc = B.grads_chunked(*_args(x, dO), dF)
    for name, a, c in zip("dq dk dv dg dbeta dA_log ddt_bias dS0".split(), ga, gc):
        assert oracle.rel_l2(c.reshape(a.shape), a) < 1e-10, name
