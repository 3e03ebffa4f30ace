"""The fp64 oracle against facts fixed by the pages and by mathematics (CPU only)."""
import json
import os

import numpy as np
import pytest

import oracle
from tests import oracle_pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kda_worked_examples.json")


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    assert pin(oracle.kda_forward) < oracle_pins.TOL


def test_hand_worked_examples():
    """Cases worked by hand from the KDA update (section 2.3), stored with their arithmetic."""
    cases = json.load(open(GOLDEN))["cases"]
    for c in cases:
        T = len(c["beta"])
        dk, dv = c["dk"], c["dv"]
        q = np.array(c["q"], float).reshape(1, T, 1, dk)
        k = np.array(c["k"], float).reshape(1, T, 1, dk)
        v = np.array(c["v"], float).reshape(1, T, 1, dv)
        g = np.log(np.array(c["a"], float)).reshape(1, T, 1, dk)
        beta = np.array(c["beta"], float).reshape(1, T, 1)
        S0 = np.array(c["S0"], float).reshape(1, 1, dk, dv)
        o, sT = oracle.kda_forward(q, k, v, g, beta, c["scale"], S0)
        np.testing.assert_allclose(o.reshape(T, dv), np.array(c["o"]), rtol=0, atol=1e-12, err_msg=c["name"])
        np.testing.assert_allclose(sT.reshape(dk, dv), np.array(c["S_final"]), rtol=0, atol=1e-12,
                                   err_msg=c["name"])


def test_boundedness():
    """With ||k|| = 1, beta in [0, 1] and a < 1, (I - b k k^T) Diag(a) is a
    contraction in the spectral norm, so ||S_t|| <= ||S_{t-1}|| + b ||v_t||."""
    rng = np.random.default_rng(11)
    dk, dv, T = 6, 4, 200
    S = rng.standard_normal((1, 1, dk, dv))
    for _ in range(T):
        k = rng.standard_normal((1, 1, 1, dk))
        k /= np.linalg.norm(k)
        q = rng.standard_normal((1, 1, 1, dk))
        v = 3 * rng.standard_normal((1, 1, 1, dv))
        g = -np.abs(rng.standard_normal((1, 1, 1, dk)))
        beta = rng.uniform(0, 1, (1, 1, 1))
        _, S1 = oracle.kda_forward(q, k, v, g, beta, 1.0, S)
        assert np.linalg.norm(S1[0, 0], 2) <= np.linalg.norm(S[0, 0], 2) + beta.item() * np.linalg.norm(v) + 1e-12
        S = S1


def test_split_sequence_equals_whole():
    """Passing the final state of a prefix as the initial state of the rest is
    the same computation (the state is the whole memory of the recurrence)."""
    rng = np.random.default_rng(12)
    B, T, H, dk, dv = 2, 37, 3, 8, 6
    q, k, v, g, beta, S0 = oracle_pins._inputs(12, B, T, H, dk, dv)
    o, sT = oracle.kda_forward(q, k, v, g, beta, 0.4, S0)
    cut = 15
    sl = lambda x, a, b: x[:, a:b]
    o1, s1 = oracle.kda_forward(*(sl(x, 0, cut) for x in (q, k, v, g, beta)), 0.4, S0)
    o2, s2 = oracle.kda_forward(*(sl(x, cut, T) for x in (q, k, v, g, beta)), 0.4, s1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s2, sT, rtol=0, atol=1e-12)


def test_decode_matches_forward():
    rng = np.random.default_rng(13)
    S, N, H, dk, dv = 5, 3, 2, 4, 7
    q, k, v, g, beta, S0 = oracle_pins._inputs(13, N, S, H, dk, dv)
    o, sT = oracle.kda_forward(q, k, v, g, beta, 0.9, S0)
    sw = lambda x: np.swapaxes(x, 0, 1)
    od, sd = oracle.kda_decode(sw(q), sw(k), sw(v), sw(g), sw(beta), 0.9, S0)
    np.testing.assert_allclose(sw(od), o, rtol=0, atol=0)
    np.testing.assert_allclose(sd, sT, rtol=0, atol=0)


def test_thread_count_does_not_change_result():
    q, k, v, g, beta, S0 = oracle_pins._inputs(14, 2, 20, 3, 8, 40)
    o1, s1 = oracle.kda_forward(q, k, v, g, beta, 0.3, S0, nthreads=1)
    o4, s4 = oracle.kda_forward(q, k, v, g, beta, 0.3, S0, nthreads=4)
    assert np.array_equal(o1, o4) and np.array_equal(s1, s4)


def test_empty_sequence_and_zero_initial_state():
    q, k, v, g, beta, S0 = oracle_pins._inputs(15, 1, 3, 1, 4, 4)
    o, sT = oracle.kda_forward(q[:, :0], k[:, :0], v[:, :0], g[:, :0], beta[:, :0], 1.0, S0)
    assert o.shape == (1, 0, 1, 4)
    np.testing.assert_array_equal(sT, S0)
    o, sT = oracle.kda_forward(q, k, v, g, beta, 1.0, None)
    o2, sT2 = oracle.kda_forward(q, k, v, g, beta, 1.0, np.zeros_like(S0))
    np.testing.assert_array_equal(o, o2)


def test_rejects_bad_mode():
    q, k, v, g, beta, S0 = oracle_pins._inputs(16, 1, 3, 1, 4, 4)
    with pytest.raises(ValueError):
        oracle.kda_forward(q, k, v, g, beta, 1.0, S0, mode=7)
