"""The oracle's chain rule through the input preparation (oracle.prepare_backward),
pinned by central differences of oracle.prepare_inputs alone and of the whole
forward (preparation, then the fp64 recurrence) along random directions."""
import numpy as np
import pytest

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


@pytest.mark.parametrize("prep", [oracle.PREP_L2NORM_QK, oracle.PREP_GATE_LOGSIGMOID, oracle.PREP_BETA_SIGMOID,
                                  oracle.PREP_L2NORM_QK | oracle.PREP_GATE_LOGSIGMOID | oracle.PREP_BETA_SIGMOID])
def test_chain_rule_matches_central_differences_of_the_preparation(prep):
    r = _rng(1)
    shp = (1, 7, 2, 16)
    q, k, g = r.standard_normal(shp), r.standard_normal(shp), 3 + r.standard_normal(shp)
    beta = r.standard_normal(shp[:3])
    w = [r.standard_normal(shp), r.standard_normal(shp), r.standard_normal(shp), r.standard_normal(shp[:3])]
    d = [r.standard_normal(shp), r.standard_normal(shp), r.standard_normal(shp), r.standard_normal(shp[:3])]

    def f(eps):
        out = oracle.prepare_inputs(q + eps * d[0], k + eps * d[1], g + eps * d[2], beta + eps * d[3], prep)
        return sum(float(np.sum(wi * oi)) for wi, oi in zip(w, out))

    eps = 1e-6
    fd = (f(eps) - f(-eps)) / (2 * eps)
    grads = oracle.prepare_backward(q, k, g, beta, prep, *w)
    dot = sum(float(np.sum(gi * di)) for gi, di in zip(grads, d))
    assert abs(fd - dot) <= 1e-7 * (1 + abs(dot)), (fd, dot)


def test_no_bits_pass_gradients_through():
    r = _rng(2)
    shp = (1, 3, 1, 8)
    x = [r.standard_normal(shp) for _ in range(3)] + [r.standard_normal(shp[:3])]
    w = [r.standard_normal(shp) for _ in range(3)] + [r.standard_normal(shp[:3])]
    for gi, wi in zip(oracle.prepare_backward(*x, 0, *w), w):
        assert np.array_equal(gi, wi)


def test_whole_forward_with_preparation_matches_central_differences():
    """L = <dO, o> + <dS_T, S_T> of the forward on prepared raw inputs: the
    chain rule after oracle.kda_backward equals its central difference."""
    r = _rng(3)
    B, T, H, D = 1, 20, 2, 8
    prep = oracle.PREP_L2NORM_QK | oracle.PREP_GATE_LOGSIGMOID | oracle.PREP_BETA_SIGMOID
    q, k, v = r.standard_normal((B, T, H, D)), r.standard_normal((B, T, H, D)), r.standard_normal((B, T, H, D))
    g, beta = 3 + r.standard_normal((B, T, H, D)), r.standard_normal((B, T, H))
    s0 = 0.1 * r.standard_normal((B, H, D, D))
    d_o, d_s = r.standard_normal((B, T, H, D)), r.standard_normal((B, H, D, D))
    scale = D ** -0.5
    dirs = [r.standard_normal(x.shape) for x in (q, k, g, beta)]

    def loss(eps):
        qp, kp, gp, bp = oracle.prepare_inputs(q + eps * dirs[0], k + eps * dirs[1], g + eps * dirs[2],
                                               beta + eps * dirs[3], prep)
        o, s = oracle.kda_forward(qp, kp, v, gp, bp, scale, s0)
        return float(np.sum(o * d_o) + np.sum(s * d_s))

    eps = 1e-6
    fd = (loss(eps) - loss(-eps)) / (2 * eps)
    qp, kp, gp, bp = oracle.prepare_inputs(q, k, g, beta, prep)
    gr = oracle.kda_backward(qp, kp, v, gp, bp, scale, s0, d_o, d_s)
    raw = oracle.prepare_backward(q, k, g, beta, prep, gr["dq"], gr["dk"], gr["dg"], gr["dbeta"])
    dot = sum(float(np.sum(gi * di)) for gi, di in zip(raw, dirs))
    assert abs(fd - dot) <= 1e-6 * (1 + abs(dot)), (fd, dot)
