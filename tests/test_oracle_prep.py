"""Pins for the oracle's fused input preparation (oracle.prepare_inputs):
closed forms, special values and a second formula for each step."""
import math

import numpy as np

import oracle


def _rng():
    return np.random.default_rng(123)


def test_l2norm_gives_unit_rows():
    r = _rng()
    q = r.normal(size=(2, 5, 3, 16)) * 7.0
    k = r.normal(size=(2, 5, 3, 16))
    qn, kn, _, _ = oracle.prepare_inputs(q, k, None, np.zeros((2, 5, 3)), oracle.PREP_L2NORM_QK)
    nq = np.sqrt((q * q).sum(-1))
    # |x / sqrt(|x|^2 + eps)| = |x| / sqrt(|x|^2 + eps), and the direction is kept
    assert np.allclose(np.linalg.norm(qn, axis=-1), nq / np.sqrt(nq * nq + 1e-6), rtol=0, atol=1e-15)
    assert np.allclose(qn * nq[..., None], q * (nq / np.sqrt(nq * nq + 1e-6))[..., None], atol=1e-12)
    assert np.allclose(np.linalg.norm(kn, axis=-1), 1.0, atol=1e-5)


def test_l2norm_of_zero_row_is_zero():
    q = np.zeros((1, 1, 1, 8))
    qn, _, _, _ = oracle.prepare_inputs(q, q, None, np.zeros((1, 1, 1)), oracle.PREP_L2NORM_QK)
    assert np.all(qn == 0.0)


def test_logsigmoid_special_values_and_second_formula():
    x = np.array([0.0, 1.0, -1.0, 3.0, -20.0, 30.0, -700.0, 700.0])
    _, _, g, _ = oracle.prepare_inputs(x, x, x, x, oracle.PREP_GATE_LOGSIGMOID)
    assert g[0] == -math.log(2.0)
    mid = np.abs(x) <= 3  # where the direct formula is itself accurate
    assert np.allclose(g[mid], np.log(1.0 / (1.0 + np.exp(-x[mid]))), rtol=1e-14, atol=0)
    assert math.isclose(g[5], -math.exp(-30.0), rel_tol=1e-12)   # log(1 + e^-x) = e^-x (1 - e^-x / 2 + ...)
    assert math.isclose(g[4], -20.0 - math.log1p(math.exp(-20.0)), rel_tol=1e-15)
    assert g[6] == -700.0                        # log sigmoid(x) -> x for x -> -inf
    assert 0.0 > g[7] > -1e-300                   # -> -e^-x for x -> +inf
    assert np.all(g <= 0.0)


def test_sigmoid_symmetry_and_values():
    x = np.linspace(-8, 8, 33)
    _, _, _, b = oracle.prepare_inputs(x, x, None, x, oracle.PREP_BETA_SIGMOID)
    assert b[16] == 0.5
    assert np.allclose(b + b[::-1], 1.0, atol=1e-15)         # sigma(-x) = 1 - sigma(x)
    assert np.allclose(b, 0.5 * (1.0 + np.tanh(0.5 * x)), rtol=1e-14)


def test_no_bits_is_identity_and_bits_are_independent():
    r = _rng()
    q, k, g, b = (r.normal(size=(1, 4, 2, 8)), r.normal(size=(1, 4, 2, 8)), r.normal(size=(1, 4, 2, 8)),
                  r.normal(size=(1, 4, 2)))
    out = oracle.prepare_inputs(q, k, g, b, 0)
    for a, e in zip(out, (q, k, g, b)):
        assert np.array_equal(a, e)
    only_beta = oracle.prepare_inputs(q, k, g, b, oracle.PREP_BETA_SIGMOID)
    assert np.array_equal(only_beta[0], q) and np.array_equal(only_beta[2], g)
