"""The chunk algebra the CUDA kernels implement, restated in numpy fp64 and
checked against the oracle's plain token-by-token recurrence (KimiLinear
article, section 2.3 for the update, sections 3.1-3.2 for the chunkwise
evaluation with its C x C per-chunk matrices).

Nothing here is the oracle and nothing here runs on a GPU: these tests pin
the derivation (the equations the kernels evaluate, in the same factored
form) so that a slip in the algebra shows up on the CPU, independently of
the CUDA code.  Per chunk of C tokens with entering state S0, G the in-chunk
inclusive cumsum of g, r a reference token:

    K+_r = k e^{G-G_r}, K-_r = k e^{G_r-G}, Q+_r = scale q e^{G-G_r}
    A_kk = diag(beta) strict_tril(K+_r K-_r^T), A_qk = tril(Q+_r K-_r^T)
    T = (I + A_kk)^-1, W = T diag(beta) K+ (K+ = k e^G), U = T diag(beta) V
    V' = U - W S0, O = Q+ S0 + A_qk V' (Q+ = scale q e^G)
    S_C = diag(e^{G_C}) S0 + Kbar^T V' (Kbar = k e^{G_C - G})

and the reverse-mode equations of the backward (dV', dS0, dAqk, dT, dA, ...).
"""
import numpy as np
import pytest

import oracle

C = 64


def _inputs(seed, B=1, T=150, H=2, dk=16, dv=8, strong=False):
    r = np.random.default_rng(seed)
    q = r.standard_normal((B, T, H, dk))
    k = r.standard_normal((B, T, H, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((B, T, H, dv))
    beta = 1.0 / (1.0 + np.exp(-r.standard_normal((B, T, H))))
    x = r.standard_normal((B, T, H, dk)) + (0.0 if strong else 3.0)
    g = np.minimum(x, 0.0) - np.log1p(np.exp(-np.abs(x)))  # log sigmoid
    s0 = 0.1 * r.standard_normal((B, H, dk, dv))
    return q, k, v, g, beta, s0


def _chunk(x, t0, nv, width):
    """Rows t0 .. t0+nv of a [T, width] slab, zero-padded to C rows."""
    out = np.zeros((C, width))
    out[:nv] = x[t0:t0 + nv]
    return out


def _chunk_operands(K, Q, V, g, bt, scale, ref):
    G = np.cumsum(g, 0)
    Gr = G[ref]
    Kpr, Kmr, Qpr = K * np.exp(G - Gr), K * np.exp(Gr - G), scale * Q * np.exp(G - Gr)
    Akk = bt[:, None] * np.tril(Kpr @ Kmr.T, -1)
    Aqk = np.tril(Qpr @ Kmr.T)
    T = np.linalg.inv(np.eye(C) + Akk)
    Kp, Qp = K * np.exp(G), scale * Q * np.exp(G)
    W = T @ (bt[:, None] * Kp)
    U = T @ (bt[:, None] * V)
    Kb = K * np.exp(G[-1] - G)
    return dict(G=G, Gr=Gr, Kpr=Kpr, Kmr=Kmr, Qpr=Qpr, Akk=Akk, Aqk=Aqk, T=T, Kp=Kp, Qp=Qp, W=W, U=U, Kb=Kb,
                gam=np.exp(G[-1]))


def chunk_forward(q, k, v, g, beta, scale, s0, ref=31):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    sT = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = s0[b, h].copy()
            for t0 in range(0, T, C):
                nv = min(C, T - t0)
                K, Q, V = _chunk(k[b, :, h], t0, nv, dk), _chunk(q[b, :, h], t0, nv, dk), _chunk(v[b, :, h], t0, nv, dv)
                c = _chunk_operands(K, Q, V, _chunk(g[b, :, h], t0, nv, dk), _chunk(beta[b, :, h, None], t0, nv, 1)[:, 0],
                                    scale, ref)
                Vp = c["U"] - c["W"] @ S
                o[b, t0:t0 + nv, h] = (c["Qp"] @ S + c["Aqk"] @ Vp)[:nv]
                S = c["gam"][:, None] * S + c["Kb"].T @ Vp
            sT[b, h] = S
    return o, sT


def chunk_backward(q, k, v, g, beta, scale, s0, d_o, d_sT, ref=31):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v), dg=np.zeros_like(g),
               dbeta=np.zeros_like(beta), dS0=np.zeros((B, H, dk, dv)))
    for b in range(B):
        for h in range(H):
            recs = []
            for t0 in range(0, T, C):
                nv = min(C, T - t0)
                K, Q, V = _chunk(k[b, :, h], t0, nv, dk), _chunk(q[b, :, h], t0, nv, dk), _chunk(v[b, :, h], t0, nv, dv)
                bt = _chunk(beta[b, :, h, None], t0, nv, 1)[:, 0]
                c = _chunk_operands(K, Q, V, _chunk(g[b, :, h], t0, nv, dk), bt, scale, ref)
                c.update(K=K, Q=Q, V=V, bt=bt, dO=_chunk(d_o[b, :, h], t0, nv, dv), t0=t0, nv=nv)
                recs.append(c)
            S = s0[b, h].copy()  # forward replay: the state entering each chunk and V'
            for c in recs:
                c["S0"] = S.copy()
                c["Vp"] = c["U"] - c["W"] @ S
                S = c["gam"][:, None] * S + c["Kb"].T @ c["Vp"]
            dS = d_sT[b, h].copy()  # reverse sweep of the state gradient
            for c in reversed(recs):
                c["dS"] = dS.copy()
                c["dVp"] = c["Aqk"].T @ c["dO"] + c["Kb"] @ dS
                dS = c["gam"][:, None] * dS + c["Qp"].T @ c["dO"] - c["W"].T @ c["dVp"]
            out["dS0"][b, h] = dS
            for c in recs:  # local gradients of each chunk
                bt, Tm, G = c["bt"], c["T"], c["G"]
                dAqk = np.tril(c["dO"] @ c["Vp"].T)
                dQs = c["dO"] @ c["S0"].T
                dW = -c["dVp"] @ c["S0"].T
                dKb = c["Vp"] @ c["dS"].T
                dT = c["dVp"] @ (bt[:, None] * c["V"]).T + dW @ (bt[:, None] * c["Kp"]).T
                dA = np.tril(-Tm.T @ dT @ Tm.T, -1)
                Xu, Xw = Tm.T @ c["dVp"], Tm.T @ dW
                P = np.tril(c["Kpr"] @ c["Kmr"].T, -1)
                dbeta = (Xu * c["V"]).sum(1) + (Xw * c["Kp"]).sum(1) + (dA * P).sum(1)
                M = bt[:, None] * dA
                dQpr = dAqk @ c["Kmr"]
                dKmr = dAqk.T @ c["Qpr"] + M.T @ c["Kpr"]
                dKpr = M @ c["Kmr"]
                ex, ei, gm, kbf = np.exp(G - c["Gr"]), np.exp(c["Gr"] - G), np.exp(G), np.exp(G[-1] - G)
                dq = scale * (ex * dQpr + gm * dQs)
                dk_ = bt[:, None] * Xw * gm + ei * dKmr + ex * dKpr + kbf * dKb
                dG = (bt[:, None] * Xw * c["Kp"] + dQpr * c["Qpr"] + dQs * c["Qp"] - dKmr * c["Kmr"] + dKpr * c["Kpr"]
                      - dKb * c["Kb"])
                dG[-1] += (dKb * c["Kb"]).sum(0) + c["gam"] * (c["dS"] * c["S0"]).sum(1)
                dg = np.cumsum(dG[::-1], 0)[::-1]
                t0, nv = c["t0"], c["nv"]
                out["dq"][b, t0:t0 + nv, h] = dq[:nv]
                out["dk"][b, t0:t0 + nv, h] = dk_[:nv]
                out["dv"][b, t0:t0 + nv, h] = (bt[:, None] * Xu)[:nv]
                out["dg"][b, t0:t0 + nv, h] = dg[:nv]
                out["dbeta"][b, t0:t0 + nv, h] = dbeta[:nv]
    return out


def _rel(a, b):
    return np.abs(a - b).max() / np.abs(b).max()


@pytest.mark.parametrize("T,dk,dv", [(150, 16, 8), (64, 8, 16), (200, 16, 16)])
def test_chunk_forward_equals_the_recurrence(T, dk, dv):
    q, k, v, g, beta, s0 = _inputs(1, T=T, dk=dk, dv=dv)
    scale = dk ** -0.5
    o_ref, s_ref = oracle.kda_forward(q, k, v, g, beta, scale, s0)
    o, s = chunk_forward(q, k, v, g, beta, scale, s0)
    assert _rel(o, o_ref) < 1e-12 and _rel(s, s_ref) < 1e-12


def test_reference_token_does_not_change_the_result():
    q, k, v, g, beta, s0 = _inputs(2)
    scale = 0.25
    o31, s31 = chunk_forward(q, k, v, g, beta, scale, s0, ref=31)
    o7, s7 = chunk_forward(q, k, v, g, beta, scale, s0, ref=7)
    assert _rel(o7, o31) < 1e-12 and _rel(s7, s31) < 1e-12


def test_w_from_the_factored_keys_scaled_per_channel():
    """W = T diag(beta) K+ equals (T diag(beta) K+_r) scaled by e^{G_r} per
    channel: the W product can run on the factored keys."""
    q, k, v, g, beta, _ = _inputs(3)
    K, Q, V = _chunk(k[0, :, 0], 0, C, 16), _chunk(q[0, :, 0], 0, C, 16), _chunk(v[0, :, 0], 0, C, 8)
    bt = beta[0, :C, 0]
    c = _chunk_operands(K, Q, V, g[0, :C, 0], bt, 0.25, 31)
    W_r = (c["T"] @ (bt[:, None] * c["Kpr"])) * np.exp(c["Gr"])[None, :]
    assert _rel(W_r, c["W"]) < 1e-13


def test_group_state_map_is_affine():
    """Over a group of chunks the state map is S_end = M S_start + R, with R
    the run from a zero start and M the run from the identity with U = 0 (the
    chunk-parallel scan's transition and offset)."""
    q, k, v, g, beta, s0 = _inputs(4, T=3 * C, dk=16, dv=16)
    scale = 0.25

    def run(S, zero_u):
        for t0 in range(0, 3 * C, C):
            K, Q, V = _chunk(k[0, :, 0], t0, C, 16), _chunk(q[0, :, 0], t0, C, 16), _chunk(v[0, :, 0], t0, C, 16)
            c = _chunk_operands(K, Q, V, g[0, t0:t0 + C, 0], beta[0, t0:t0 + C, 0], scale, 31)
            Vp = (0.0 if zero_u else c["U"]) - c["W"] @ S
            S = c["gam"][:, None] * S + c["Kb"].T @ Vp
        return S

    R = run(np.zeros((16, 16)), False)
    M = run(np.eye(16), True)
    assert _rel(M @ s0[0, 0] + R, run(s0[0, 0], False)) < 1e-12


def test_chunk_backward_equals_the_oracle_gradients():
    q, k, v, g, beta, s0 = _inputs(5)
    r = np.random.default_rng(6)
    d_o, d_sT = r.standard_normal(v.shape), r.standard_normal(s0.shape)
    scale = 0.25
    ref = oracle.kda_backward(q, k, v, g, beta, scale, s0, d_o, d_sT)
    got = chunk_backward(q, k, v, g, beta, scale, s0, d_o, d_sT)
    for n in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        assert _rel(got[n], ref[n]) < 1e-10, n


def test_chunk_backward_with_strong_decay():
    """Gates near log sigmoid(N(0,1)): the factors e^{G-G_r} span a wide range
    inside a chunk (still inside the factored form's safe span)."""
    q, k, v, g, beta, s0 = _inputs(7, T=100, strong=True)
    r = np.random.default_rng(8)
    d_o, d_sT = r.standard_normal(v.shape), r.standard_normal(s0.shape)
    ref = oracle.kda_backward(q, k, v, g, beta, 0.25, s0, d_o, d_sT)
    got = chunk_backward(q, k, v, g, beta, 0.25, s0, d_o, d_sT)
    for n in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        assert _rel(got[n], ref[n]) < 1e-9, n


@pytest.mark.parametrize("gate", ["head", "none"])
def test_scalar_gate_forms(gate):
    """Gated DeltaNet (one log-gate per token and head, broadcast over the key
    channels) and DeltaNet (no forgetting, g = 0) through the same chunk
    equations."""
    q, k, v, g, beta, s0 = _inputs(9, T=130)
    g = np.repeat(g[..., :1], g.shape[-1], axis=-1) if gate == "head" else np.zeros_like(g)
    o_ref, s_ref = oracle.kda_forward(q, k, v, g, beta, 0.25, s0)
    o, s = chunk_forward(q, k, v, g, beta, 0.25, s0)
    assert _rel(o, o_ref) < 1e-12 and _rel(s, s_ref) < 1e-12


def test_exact_pairwise_form_equals_the_factored_one():
    """The kernels' exact path forms every decay factor e^{G_i - G_j} (<= 1
    for j <= i) per pair and channel instead of factoring it around G_r."""
    q, k, v, g, beta, _ = _inputs(10, strong=True)
    K, Q, V = _chunk(k[0, :, 0], 0, C, 16), _chunk(q[0, :, 0], 0, C, 16), _chunk(v[0, :, 0], 0, C, 8)
    bt = beta[0, :C, 0]
    c = _chunk_operands(K, Q, V, g[0, :C, 0], bt, 0.25, 31)
    G = c["G"]
    E = np.exp(G[:, None, :] - G[None, :, :])  # [i, j, channel]
    Akk = bt[:, None] * np.tril(np.einsum("ic,jc,ijc->ij", K, K, E), -1)
    Aqk = np.tril(0.25 * np.einsum("ic,jc,ijc->ij", Q, K, E))
    assert np.all(np.tril(E.max(axis=2)) <= 1.0 + 1e-15)
    assert _rel(Akk, c["Akk"]) < 1e-12 and _rel(Aqk, c["Aqk"]) < 1e-12


def _bf16(x):
    """Round to the nearest bf16 (ties to even), returned as float64."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def test_bf16_rounding_points_meet_the_tolerance():
    """The bf16 prefill's precision plan: inputs in bf16; the chunk operands
    (K+_r, Q+_r, K-_r, T diag(beta), V, and the records -W, Q+, A_qk, Kbar, U)
    rounded to bf16 where they enter tensor-core products; the state kept in
    fp32 and rounded to bf16 only as an operand (S0 in P and O, V' in the
    update); fp32 accumulation.  Over a 16-chunk chain at d = 128 the outputs
    and the final state stay inside the 1e-2 bound against the fp64
    recurrence on the same bf16 inputs (about 6e-3 for o and 4e-3 for the
    state here, the range the GPU kernels measure)."""
    r = np.random.default_rng(11)
    T, d = 16 * C, 128
    q = r.standard_normal((T, d))
    k = r.standard_normal((T, d))
    q = _bf16(q / np.linalg.norm(q, axis=-1, keepdims=True))
    k = _bf16(k / np.linalg.norm(k, axis=-1, keepdims=True))
    v = _bf16(r.standard_normal((T, d)))
    beta = _bf16(1.0 / (1.0 + np.exp(-r.standard_normal(T))))
    x = r.standard_normal((T, d)) + 3.0
    g = _bf16(np.minimum(x, 0.0) - np.log1p(np.exp(-np.abs(x))))
    s0 = 0.1 * r.standard_normal((d, d))
    scale = d ** -0.5
    f32 = lambda a: np.asarray(a, dtype=np.float32).astype(np.float64)
    S = s0.copy()
    o = np.zeros((T, d))
    for t0 in range(0, T, C):
        K, Q, V, bt = k[t0:t0 + C], q[t0:t0 + C], v[t0:t0 + C], beta[t0:t0 + C]
        G = f32(np.cumsum(g[t0:t0 + C], 0))
        Gr = G[31]
        Kpr, Kmr, Qpr = _bf16(K * np.exp(G - Gr)), _bf16(K * np.exp(Gr - G)), _bf16(scale * Q * np.exp(G - Gr))
        Akk = f32(bt[:, None] * np.tril(f32(Kpr @ Kmr.T), -1))
        Aqk = _bf16(np.tril(f32(Qpr @ Kmr.T)))
        TB = _bf16(np.linalg.inv(np.eye(C) + Akk) * bt[None, :])  # (T diag beta), fp32 solve, bf16 operand
        Wm = _bf16(-f32(TB @ Kpr) * np.exp(Gr)[None, :])             # -W record
        U = _bf16(f32(TB @ V))
        Qp = _bf16(scale * Q * np.exp(G))
        Kb = _bf16(K * np.exp(G[-1] - G))
        gam = f32(np.exp(G[-1]))
        Sb = _bf16(S)
        Vp = _bf16(f32(U + f32(Wm @ Sb)))
        o[t0:t0 + C] = f32(f32(Qp @ Sb) + f32(Aqk @ Vp))
        S = f32(gam[:, None] * S + f32(Kb.T @ Vp))
    o_ref, s_ref = oracle.kda_forward(q[None, :, None], k[None, :, None], v[None, :, None], g[None, :, None],
                                      beta[None, :, None], scale, s0[None, None])
    eo, es = _rel(o, o_ref[0, :, 0]), _rel(S, s_ref[0, 0])
    assert eo < 1e-2 and es < 1e-2, (eo, es)
    assert eo > 1e-4 and es > 1e-4, (eo, es)  # the rounding is really applied
