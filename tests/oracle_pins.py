"""Pins for the fp64 KDA oracle: facts fixed by the KimiLinear pages and by
mathematics, each computed WITHOUT the oracle's own loops.

Every pin is a function ``pin_*(fwd) -> float`` returning an error that must be
below ``TOL``; ``fwd`` has the signature of ``oracle.kda_forward``.  The same
functions run against the real oracle (tests/test_oracle_pins.py) and against
deliberately broken copies of it (tests/test_oracle_mutants.py), which shows
that a plausible slip in the oracle fails at least one pin.

Sources of the facts (KimiLinear: A Next-Generation Linear Attention
Architecture for Long-Context LLMs):
  section 2.1  linear attention  S_t = S_{t-1} + v k^T;  DeltaNet
               S_t = (I - b k k^T) S_{t-1} + b v k^T, and b -> 1 overwrites;
  section 2.2  Gated DeltaNet    S_t = a_t (I - b k k^T) S_{t-1} + b v k^T;
  section 2.3  KDA               S_t = (I - b k k^T) Diag(a_t) S_{t-1} + b v k^T,
               a_t acting on the rows of the state.
All formulas are used in the d_k x d_v orientation (write term k v^T,
output o = scale S^T q).
"""
from __future__ import annotations

import numpy as np

TOL = 1e-10


def _rng(seed):
    return np.random.default_rng(seed)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _inputs(seed, B, T, H, dk, dv, gate="random", s0=True, unit_k=True):
    r = _rng(seed)
    q = _unit(r.standard_normal((B, T, H, dk)))
    k = r.standard_normal((B, T, H, dk))
    if unit_k:
        k = _unit(k)
    v = r.standard_normal((B, T, H, dv))
    beta = 1.0 / (1.0 + np.exp(-r.standard_normal((B, T, H))))
    if gate == "random":
        g = -np.log1p(np.exp(-(r.standard_normal((B, T, H, dk)) + 1.0)))  # logsigmoid(N(1,1))
    elif gate == "zero":
        g = np.zeros((B, T, H, dk))
    elif gate == "scalar":
        g = np.repeat(-np.log1p(np.exp(-(r.standard_normal((B, T, H, 1)) + 1.0))), dk, axis=-1)
    else:
        raise ValueError(gate)
    S0 = 0.3 * r.standard_normal((B, H, dk, dv)) if s0 else None
    return q, k, v, g, beta, S0


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(1e-300, np.max(np.abs(b))))


def pin_linear_attention_closed_form(fwd):
    """Plain linear attention (section 2.1): with the delta correction off,
    a = 1 and b = 1 the state is a running sum of k v^T, so the outputs are the
    masked product O = scale (tril(Q K^T) V + Q S0) and S_T = S0 + K^T V."""
    import oracle
    B, T, H, dk, dv = 2, 9, 3, 5, 7
    q, k, v, _, _, S0 = _inputs(1, B, T, H, dk, dv, unit_k=False)
    g = np.zeros((B, T, H, dk))
    beta = np.ones((B, T, H))
    scale = 0.37
    o, sT = fwd(q, k, v, g, beta, scale, S0, mode=oracle.MODE_LINEAR)
    err = 0.0
    mask = np.tril(np.ones((T, T)))
    for b in range(B):
        for h in range(H):
            Q, K, V = q[b, :, h], k[b, :, h], v[b, :, h]
            O = scale * ((Q @ K.T) * mask) @ V + scale * Q @ S0[b, h]
            err = max(err, _rel(o[b, :, h], O), _rel(sT[b, h], S0[b, h] + K.T @ V))
    return err


def pin_gated_linear_closed_form(fwd):
    """Gated linear attention (delta correction off, per-channel gates on the
    rows): unrolling S_t = Diag(a_t) S_{t-1} + b_t k_t v_t^T gives
    S_t = Diag(G_t) S0 + sum_{s<=t} Diag(G_t / G_s) k_s b_s v_s^T with
    G_t = prod_{r<=t} a_r.  Computed here with explicit pairwise decay
    factors; pins the gate axis, the decay-before-write order and the output
    read after the write."""
    import oracle
    B, T, H, dk, dv = 1, 11, 2, 4, 6
    q, k, v, g, beta, S0 = _inputs(2, B, T, H, dk, dv, unit_k=False)
    scale = 0.81
    o, sT = fwd(q, k, v, g, beta, scale, S0, mode=oracle.MODE_LINEAR)
    err = 0.0
    for b in range(B):
        for h in range(H):
            logG = np.cumsum(g[b, :, h], axis=0)  # [T, dk]
            for t in range(T):
                St = np.exp(logG[t])[:, None] * S0[b, h]
                for s in range(t + 1):
                    dec = np.exp(logG[t] - logG[s])
                    St = St + np.outer(dec * k[b, s, h], beta[b, s, h] * v[b, s, h])
                err = max(err, _rel(o[b, t, h], scale * St.T @ q[b, t, h]))
            err = max(err, _rel(sT[b, h], St))
    return err


def _transition(k, g, beta):
    dk = k.shape[0]
    return (np.eye(dk) - beta * np.outer(k, k)) @ np.diag(np.exp(g))


def pin_brute_force_products(fwd):
    """KDA (section 2.3) unrolled: S_t = (A_t...A_1) S0 + sum_{s<=t}
    (A_t...A_{s+1}) b_s k_s v_s^T with the dense transition
    A_s = (I - b_s k_s k_s^T) Diag(exp g_s).  Every S_t is rebuilt from the
    explicit matrix products (no recursion on S), for T <= 8, d_k != d_v and
    a value width that spans several of the oracle's column blocks."""
    B, T, H, dk, dv = 2, 8, 2, 6, 19
    q, k, v, g, beta, S0 = _inputs(3, B, T, H, dk, dv)
    scale = 0.6
    o, sT = fwd(q, k, v, g, beta, scale, S0)
    err = 0.0
    for b in range(B):
        for h in range(H):
            A = [_transition(k[b, s, h], g[b, s, h], beta[b, s, h]) for s in range(T)]
            for t in range(T):
                P = np.eye(dk)
                for s in range(t, -1, -1):
                    P = P @ A[s]
                St = P @ S0[b, h]
                for s in range(t + 1):
                    P = np.eye(dk)
                    for r in range(t, s, -1):
                        P = P @ A[r]
                    St = St + P @ np.outer(beta[b, s, h] * k[b, s, h], v[b, s, h])
                err = max(err, _rel(o[b, t, h], scale * St.T @ q[b, t, h]))
            err = max(err, _rel(sT[b, h], St))
    return err


def pin_exact_retrieval(fwd):
    """DeltaNet overwrite (section 2.1, b -> 1): with ||k_t|| = 1, b_t = 1 and
    a = 1, (I - k k^T) S k = 0, so k_t^T S_t = v_t^T exactly.  Reading with
    q_t = k_t and scale 1 must therefore return v_t."""
    B, T, H, dk, dv = 2, 40, 2, 8, 5
    _, k, v, _, _, S0 = _inputs(4, B, T, H, dk, dv)
    g = np.zeros((B, T, H, dk))
    beta = np.ones((B, T, H))
    o, _ = fwd(k, k, v, g, beta, 1.0, S0)
    return float(np.max(np.abs(o - v)))


def pin_deltanet_reduction(fwd):
    """a = 1 (g = 0) turns KDA into DeltaNet (section 2.1),
    S_t = (I - b k k^T) S_{t-1} + b k v^T, here as dense matrix algebra."""
    B, T, H, dk, dv = 1, 30, 2, 7, 9
    q, k, v, _, beta, S0 = _inputs(5, B, T, H, dk, dv)
    g = np.zeros((B, T, H, dk))
    scale = 0.5
    o, sT = fwd(q, k, v, g, beta, scale, S0)
    err = 0.0
    for h in range(H):
        S = S0[0, h].copy()
        for t in range(T):
            kk, bb = k[0, t, h], beta[0, t, h]
            S = (np.eye(dk) - bb * np.outer(kk, kk)) @ S + bb * np.outer(kk, v[0, t, h])
            err = max(err, _rel(o[0, t, h], scale * S.T @ q[0, t, h]))
        err = max(err, _rel(sT[0, h], S))
    return err


def pin_gdn_reduction(fwd):
    """A gate equal across channels turns KDA into Gated DeltaNet
    (section 2.2), S_t = a_t (I - b k k^T) S_{t-1} + b k v^T."""
    B, T, H, dk, dv = 1, 30, 2, 7, 9
    q, k, v, g, beta, S0 = _inputs(6, B, T, H, dk, dv, gate="scalar")
    scale = 0.5
    o, sT = fwd(q, k, v, g, beta, scale, S0)
    err = 0.0
    for h in range(H):
        S = S0[0, h].copy()
        for t in range(T):
            kk, bb, a = k[0, t, h], beta[0, t, h], np.exp(g[0, t, h, 0])
            S = a * (np.eye(dk) - bb * np.outer(kk, kk)) @ S + bb * np.outer(kk, v[0, t, h])
            err = max(err, _rel(o[0, t, h], scale * S.T @ q[0, t, h]))
        err = max(err, _rel(sT[0, h], S))
    return err


def pin_zero_beta_pure_decay(fwd):
    """b = 0 writes nothing: S_t = Diag(prod a) S0 exactly and
    o_t = scale S_t^T q_t."""
    B, T, H, dk, dv = 1, 12, 1, 5, 3
    q, k, v, g, _, S0 = _inputs(7, B, T, H, dk, dv)
    beta = np.zeros((B, T, H))
    o, sT = fwd(q, k, v, g, beta, 1.0, S0)
    logG = np.cumsum(g[0, :, 0], axis=0)
    err = _rel(sT[0, 0], np.exp(logG[-1])[:, None] * S0[0, 0])
    for t in range(T):
        err = max(err, _rel(o[0, t, 0], (np.exp(logG[t])[:, None] * S0[0, 0]).T @ q[0, t, 0]))
    return err


ALL_PINS = [
    pin_linear_attention_closed_form,
    pin_gated_linear_closed_form,
    pin_brute_force_products,
    pin_exact_retrieval,
    pin_deltanet_reduction,
    pin_gdn_reduction,
    pin_zero_beta_pure_decay,
]
