"""Pins for the oracle's backward pass (oracle.kda_backward): central finite
differences of the fp64 forward oracle, and reverse-mode autodiff (torch
autograd) through a plain fp64 loop of the recurrence; both on tiny shapes."""
import numpy as np
import pytest
import torch

import oracle


def _problem(seed, B=1, T=6, H=2, dk=4, dv=3):
    r = np.random.default_rng(seed)
    q = r.normal(size=(B, T, H, dk))
    k = r.normal(size=(B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.normal(size=(B, T, H, dv))
    g = -np.abs(r.normal(size=(B, T, H, dk))) * 0.5
    beta = 1.0 / (1.0 + np.exp(-r.normal(size=(B, T, H))))
    s0 = r.normal(size=(B, H, dk, dv)) * 0.3
    d_o = r.normal(size=(B, T, H, dv))
    d_s = r.normal(size=(B, H, dk, dv))
    return dict(q=q, k=k, v=v, g=g, beta=beta, s0=s0), d_o, d_s


def _loss(x, d_o, d_s, scale):
    o, s = oracle.kda_forward(x["q"], x["k"], x["v"], x["g"], x["beta"], scale, x["s0"])
    return float(np.sum(o * d_o) + np.sum(s * d_s))


@pytest.mark.parametrize("seed", [1, 2])
def test_backward_matches_finite_differences(seed):
    x, d_o, d_s = _problem(seed)
    scale = 0.7
    grads = oracle.kda_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], scale, x["s0"], d_o, d_s)
    names = {"q": "dq", "k": "dk", "v": "dv", "g": "dg", "beta": "dbeta", "s0": "dS0"}
    h = 1e-6
    for n, gname in names.items():
        a = x[n]
        fd = np.zeros_like(a)
        for idx in np.ndindex(a.shape):
            keep = a[idx]
            a[idx] = keep + h
            lp = _loss(x, d_o, d_s, scale)
            a[idx] = keep - h
            lm = _loss(x, d_o, d_s, scale)
            a[idx] = keep
            fd[idx] = (lp - lm) / (2 * h)
        err = np.max(np.abs(fd - grads[gname])) / max(1e-12, np.max(np.abs(fd)))
        assert err < 1e-6, (n, err)


def _torch_forward(q, k, v, g, beta, s0, scale):
    """The recurrence as a plain fp64 loop (for autograd only)."""
    B, T, H, dk = q.shape
    outs = []
    S = s0.clone()
    for t in range(T):
        a = torch.exp(g[:, t])                                   # [B,H,dk]
        Sp = a.unsqueeze(-1) * S                                 # decay rows
        pred = torch.einsum("bhij,bhi->bhj", Sp, k[:, t])
        u = beta[:, t].unsqueeze(-1) * (v[:, t] - pred)          # [B,H,dv]
        S = Sp + k[:, t].unsqueeze(-1) * u.unsqueeze(-2)
        outs.append(scale * torch.einsum("bhij,bhi->bhj", S, q[:, t]))
    return torch.stack(outs, dim=1), S


def test_backward_matches_autograd():
    x, d_o, d_s = _problem(3, B=2, T=9, H=1, dk=5, dv=4)
    scale = 0.45
    t = {n: torch.tensor(a, dtype=torch.float64, requires_grad=True) for n, a in x.items()}
    o, s = _torch_forward(t["q"], t["k"], t["v"], t["g"], t["beta"], t["s0"], scale)
    (torch.sum(o * torch.tensor(d_o)) + torch.sum(s * torch.tensor(d_s))).backward()
    grads = oracle.kda_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], scale, x["s0"], d_o, d_s)
    for n, gname in {"q": "dq", "k": "dk", "v": "dv", "g": "dg", "beta": "dbeta", "s0": "dS0"}.items():
        ref = t[n].grad.numpy()
        assert np.allclose(grads[gname], ref, rtol=1e-11, atol=1e-12), n


def test_backward_without_final_state_gradient():
    """dL/dS_T = 0 and dL/do = 0 give zero gradients everywhere."""
    x, d_o, _ = _problem(4)
    grads = oracle.kda_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], 1.0, x["s0"], np.zeros_like(d_o))
    for a in grads.values():
        assert np.all(a == 0.0)
