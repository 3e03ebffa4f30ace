"""Backward pass (kda_backward) against the fp64 oracle's gradients
(oracle.kda_backward, pinned by finite differences and autograd)."""
import pytest
import torch

import oracle
from gated_delta_rule_67_b200 import kda_backward
from gated_delta_rule_67_b200.workloads import make_cotangents, make_head_gates, make_prefill_inputs
from tests.parity import TOL, cuda_or_skip, rel_err

pytestmark = pytest.mark.gpu


def _case(B, T, H, dk, dv, dtype, gate="channel", s0=0.1, final=True, seed=90):
    dev = cuda_or_skip()
    x = make_prefill_inputs(B, T, H, dk, dv, dtype, s0, seed=seed)
    d_o, d_s = make_cotangents(B, T, H, dk, dv, dtype, seed=seed + 1, final_state=final)
    if gate == "head":
        g = make_head_gates((B, T, H), 1, dtype, seed=seed + 2)
        g_or = g.unsqueeze(-1).expand_as(x["q"]).contiguous()
    elif gate == "none":
        g, g_or = None, torch.zeros_like(x["q"])
    else:
        g = g_or = x["g"]
    scale = dk ** -0.5
    to = lambda t: None if t is None else t.to(dev)
    got = kda_backward(to(x["q"]), to(x["k"]), to(x["v"]), to(g), to(x["beta"]), to(d_o), scale,
                       to(x["initial_state"]), to(d_s))
    torch.cuda.synchronize()
    ref = oracle.kda_backward(x["q"], x["k"], x["v"], g_or, x["beta"], scale, x["initial_state"], d_o, d_s)
    tol = TOL[dtype]
    for name in ("dq", "dk", "dv", "dbeta", "dS0"):
        assert rel_err(got[name], ref[name]) < tol, (name, rel_err(got[name], ref[name]))
    if gate == "channel":
        assert rel_err(got["dg"], ref["dg"]) < tol, ("dg", rel_err(got["dg"], ref["dg"]))
    elif gate == "head":
        dgh = ref["dg"].sum(axis=-1)   # the per-head gate is broadcast over the key channels
        assert rel_err(got["dg"], dgh) < tol, ("dg", rel_err(got["dg"], dgh))
    else:
        assert got["dg"] is None
    return got


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("B,T,H,dk,dv", [(1, 37, 2, 128, 128), (2, 100, 3, 64, 64), (1, 64, 1, 128, 64),
                                         (1, 64, 1, 64, 128), (1, 1, 1, 128, 128), (1, 65, 2, 128, 128),
                                         (1, 200, 2, 128, 128), (2, 130, 3, 64, 128), (1, 129, 2, 128, 64)])
def test_backward_shapes(dtype, B, T, H, dk, dv):
    """One and several 64-token chunks with ragged tails (65 tokens: a
    one-token tail), a single token, every supported (dk, dv)."""
    _case(B, T, H, dk, dv, dtype, seed=91 + T)


@pytest.mark.parametrize("gate", ["head", "none"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_backward_scalar_gates(gate, dtype):
    _case(1, 150, 2, 128, 128, dtype, gate=gate, seed=92)


def test_backward_zero_state_and_no_final_gradient():
    _case(2, 70, 2, 128, 128, torch.float32, s0=0.0, final=False, seed=93)


def test_backward_bench_shape():
    """B=1, H=16, T=4096, d=128 (bf16), random initial state, every gradient."""
    _case(1, 4096, 16, 128, 128, torch.bfloat16, seed=94)


def test_backward_deterministic():
    dev = cuda_or_skip()
    x = make_prefill_inputs(1, 200, 2, 128, 128, torch.bfloat16, 0.1, seed=95, device=dev)
    d_o, d_s = make_cotangents(1, 200, 2, 128, 128, torch.bfloat16, seed=96, device=dev)
    args = (x["q"], x["k"], x["v"], x["g"], x["beta"], d_o, None, x["initial_state"], d_s)
    a, b = kda_backward(*args), kda_backward(*args)
    torch.cuda.synchronize()
    for n in a:
        assert torch.equal(a[n], b[n]), n


@pytest.mark.parametrize("B,H", [(2, 8), (5, 8)], ids=["32-columns", "64-columns"])
def test_backward_pass_widths(B, H):
    """The state passes give each CTA 32 value columns while 2 x B H x d_v/32
    CTAs fit in one wave of 148 SMs (16 pairs), else 64 (40 pairs)."""
    _case(B, 200, H, 128, 128, torch.float32, seed=97 + B)


def _extreme_gates(x, dtype):
    """Per-channel log-gates with chunks whose cumulative decay leaves the
    factored operands' safe span (|G_i - G_31| > 64): -4 per token in half
    of the channels of the second chunk, -80 at one token of the fourth."""
    g = x["g"].clone().float()
    g[:, 64:128, :, ::2] = -4.0
    g[:, 200, :, 5] = -80.0
    x["g"] = g.to(dtype)
    return x


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_backward_exact_pairwise_path(dtype):
    """Chunks past the factored form's span take the exact per-element path;
    the others in the same call keep the tensor-core path."""
    dev = cuda_or_skip()
    B, T, H, dk, dv = 1, 230, 2, 128, 128
    x = _extreme_gates(make_prefill_inputs(B, T, H, dk, dv, dtype, 0.1, seed=98), dtype)
    d_o, d_s = make_cotangents(B, T, H, dk, dv, dtype, seed=99)
    to = lambda t: t.to(dev)
    got = kda_backward(to(x["q"]), to(x["k"]), to(x["v"]), to(x["g"]), to(x["beta"]), to(d_o), dk ** -0.5,
                       to(x["initial_state"]), to(d_s))
    torch.cuda.synchronize()
    ref = oracle.kda_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], dk ** -0.5, x["initial_state"], d_o, d_s)
    for name in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        assert rel_err(got[name], ref[name]) < TOL[dtype], (name, rel_err(got[name], ref[name]))


@pytest.mark.parametrize("fit", [1, 2, 4], ids=["one-pair", "two-pairs", "four-pairs"])
def test_backward_small_workspace_groups(fit):
    """A workspace for `fit` (sequence, head) pairs processes the 6 pairs in
    groups; the result is bit-identical to the one-group call."""
    dev = cuda_or_skip()
    from gated_delta_rule_67_b200.binding import load
    B, T, H = 2, 130, 3
    x = make_prefill_inputs(B, T, H, 128, 128, torch.bfloat16, 0.1, seed=100, device=dev)
    d_o, d_s = make_cotangents(B, T, H, 128, 128, torch.bfloat16, seed=101, device=dev)
    args = (x["q"], x["k"], x["v"], x["g"], x["beta"], d_o, None, x["initial_state"], d_s)
    one = int(load().kda_backward_workspace_size(1, T, 1, 128, 128, 1))
    full = kda_backward(*args)
    part = kda_backward(*args, workspace=torch.empty(fit * one + 8, dtype=torch.uint8, device=dev))
    torch.cuda.synchronize()
    for n in full:
        assert torch.equal(full[n], part[n]), n


def test_backward_tensor_core_workspace_groups():
    """40 (sequence, head) pairs through a workspace for 20: two groups, each
    on the tensor-core path, whose preparation starts the second group at pair
    20 of the inputs; bit-identical to the one-group call."""
    dev = cuda_or_skip()
    from gated_delta_rule_67_b200.binding import load
    B, T, H = 2, 130, 20
    x = make_prefill_inputs(B, T, H, 128, 128, torch.bfloat16, 0.1, seed=102, device=dev)
    d_o, d_s = make_cotangents(B, T, H, 128, 128, torch.bfloat16, seed=103, device=dev)
    args = (x["q"], x["k"], x["v"], x["g"], x["beta"], d_o, None, x["initial_state"], d_s)
    one = int(load().kda_backward_workspace_size(1, T, 1, 128, 128, 1))
    full = kda_backward(*args)
    part = kda_backward(*args, workspace=torch.empty(20 * one + 8, dtype=torch.uint8, device=dev))
    torch.cuda.synchronize()
    for n in full:
        assert torch.equal(full[n], part[n]), n


@pytest.mark.parametrize("gate", ["channel", "head"])
def test_backward_matches_gpu_forward_directional_derivative(gate):
    """Independent of the oracle: for L = <dO, o> + <dS_T, S_T> computed from
    the library's own fp32 forward, the central difference of L along a random
    direction of (q, k, v, g, beta, S_0) equals the sum of the backward's
    gradients times that direction."""
    from gated_delta_rule_67_b200 import kda_chunk_fwd
    dev = cuda_or_skip()
    B, T, H, dk, dv = 1, 150, 2, 64, 64
    x = make_prefill_inputs(B, T, H, dk, dv, torch.float32, 0.1, seed=102, device=dev)
    if gate == "head":
        x["g"] = make_head_gates((B, T, H), 1, torch.float32, seed=103, device=dev)
    d_o, d_s = make_cotangents(B, T, H, dk, dv, torch.float32, seed=104, device=dev)
    names = ("q", "k", "v", "g", "beta", "initial_state")
    gen = torch.Generator(device="cpu").manual_seed(105)
    direction = {n: (0.1 * torch.randn(x[n].shape, generator=gen)).to(dev) for n in names}
    scale = dk ** -0.5

    def loss(eps):
        y = {n: x[n] + eps * direction[n] for n in names}
        o, s = kda_chunk_fwd(y["q"], y["k"], y["v"], y["g"], y["beta"], scale, y["initial_state"])
        torch.cuda.synchronize()
        return float((o.double() * d_o.double()).sum() + (s.double() * d_s.double()).sum())

    eps = 1e-2
    fd = (loss(eps) - loss(-eps)) / (2 * eps)
    gr = kda_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], d_o, scale, x["initial_state"], d_s)
    torch.cuda.synchronize()
    key = dict(q="dq", k="dk", v="dv", g="dg", beta="dbeta", initial_state="dS0")
    dot = sum(float((gr[key[n]].double() * direction[n].double()).sum()) for n in names)
    assert abs(fd - dot) <= 1e-3 * abs(dot) + 1e-3, (fd, dot)


@pytest.mark.parametrize("prep", [7, 1, 2, 4], ids=["all", "l2norm", "logsigmoid", "sigmoid"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_backward_through_fused_preparation(prep, dtype):
    """Raw inputs with KDA_PREP_* bits: the gradients with respect to the raw
    q, k, g, beta equal the oracle's backward on the prepared inputs followed
    by its chain rule through the preparation (oracle.prepare_backward)."""
    from gated_delta_rule_67_b200.workloads import make_raw_prefill_inputs
    dev = cuda_or_skip()
    B, T, H, dk, dv = 1, 150, 2, 128, 128
    x = make_raw_prefill_inputs(B, T, H, dk, dv, dtype, 0.1, seed=106)
    ready = make_prefill_inputs(B, T, H, dk, dv, dtype, 0.1, seed=106)  # inputs whose step is not selected
    if not prep & 1:
        x["q"], x["k"] = ready["q"], ready["k"]
    if not prep & 2:
        x["g"] = ready["g"]
    if not prep & 4:
        x["beta"] = ready["beta"]
    d_o, d_s = make_cotangents(B, T, H, dk, dv, dtype, seed=107)
    scale = dk ** -0.5
    to = lambda t: t.to(dev)
    got = kda_backward(to(x["q"]), to(x["k"]), to(x["v"]), to(x["g"]), to(x["beta"]), to(d_o), scale,
                       to(x["initial_state"]), to(d_s), prep=prep)
    torch.cuda.synchronize()
    qp, kp, gp, bp = oracle.prepare_inputs(x["q"], x["k"], x["g"], x["beta"], prep)
    ref = oracle.kda_backward(qp, kp, x["v"], gp, bp, scale, x["initial_state"], d_o, d_s)
    dq, dk_, dg, db = oracle.prepare_backward(x["q"], x["k"], x["g"], x["beta"], prep, ref["dq"], ref["dk"], ref["dg"],
                                              ref["dbeta"])
    want = dict(dq=dq, dk=dk_, dv=ref["dv"], dg=dg, dbeta=db, dS0=ref["dS0"])
    for name, r in want.items():
        assert rel_err(got[name], r) < TOL[dtype], (name, rel_err(got[name], r))


def test_backward_through_preparation_head_gate():
    """Per-head raw gates with the log-sigmoid bit (and the other two bits)."""
    dev = cuda_or_skip()
    from gated_delta_rule_67_b200.workloads import make_raw_prefill_inputs
    B, T, H, dk, dv = 1, 100, 2, 64, 64
    x = make_raw_prefill_inputs(B, T, H, dk, dv, torch.float32, 0.1, seed=108)
    gh = make_head_gates((B, T, H), 1, torch.float32, seed=109, raw=True)
    d_o, d_s = make_cotangents(B, T, H, dk, dv, torch.float32, seed=110)
    to = lambda t: t.to(dev)
    got = kda_backward(to(x["q"]), to(x["k"]), to(x["v"]), to(gh), to(x["beta"]), to(d_o), None,
                       to(x["initial_state"]), to(d_s), prep=7)
    torch.cuda.synchronize()
    g_b = gh.unsqueeze(-1).expand_as(x["q"]).contiguous()
    qp, kp, gp, bp = oracle.prepare_inputs(x["q"], x["k"], g_b, x["beta"], 7)
    ref = oracle.kda_backward(qp, kp, x["v"], gp, bp, dk ** -0.5, x["initial_state"], d_o, d_s)
    dq, dk_, dg, db = oracle.prepare_backward(x["q"], x["k"], g_b, x["beta"], 7, ref["dq"], ref["dk"], ref["dg"],
                                              ref["dbeta"])
    assert rel_err(got["dg"], dg.sum(axis=-1)) < TOL[torch.float32]
    for name, r in dict(dq=dq, dk=dk_, dv=ref["dv"], dbeta=db, dS0=ref["dS0"]).items():
        assert rel_err(got[name], r) < TOL[torch.float32], (name, rel_err(got[name], r))


def test_backward_long_chain():
    """One (sequence, head) over 65,536 tokens (1,024 chunks, bf16): the state
    passes carry the state and its gradient through the whole chain."""
    _case(1, 65536, 1, 128, 128, torch.bfloat16, seed=111)


def test_backward_error_word_and_many_waves():
    """bf16, d = 128 (the tensor-core state passes): 160 (sequence, head)
    chains x 2 roles = 320 pass CTAs (more than one wave of SMs); every
    gradient against the oracle, and the workspace's error word reads clear."""
    from gated_delta_rule_67_b200 import binding, kda_chunk_fwd_check
    dev = cuda_or_skip()
    B, T, H, d = 4, 150, 40, 128
    x = make_prefill_inputs(B, T, H, d, d, torch.bfloat16, 0.1, seed=97)
    d_o, d_s = make_cotangents(B, T, H, d, d, torch.bfloat16, seed=98)
    ws = torch.empty(int(binding.load().kda_backward_workspace_size(B, T, H, d, d, 1)), dtype=torch.uint8, device=dev)
    ws.fill_(0xCD)
    to = lambda t: t.to(dev)
    got = kda_backward(to(x["q"]), to(x["k"]), to(x["v"]), to(x["g"]), to(x["beta"]), to(d_o), None,
                       to(x["initial_state"]), to(d_s), workspace=ws)
    assert kda_chunk_fwd_check(ws) == binding.KDA_OK
    ref = oracle.kda_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], d ** -0.5, x["initial_state"], d_o, d_s)
    for name in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        assert rel_err(got[name], ref[name]) < TOL[torch.bfloat16], name


@pytest.mark.parametrize("T,gate,s0,final", [(100, "channel", 0.1, True), (64 * 3 + 7, "head", 0.1, True),
                                             (70, "none", 0.1, True), (1, "channel", 0.1, True),
                                             (130, "channel", 0.0, False)])
def test_backward_tensor_core_passes(T, gate, s0, final):
    """bf16, d = 128 with at least a wave of pass CTAs (2 x 40 heads x 2 sequences):
    the state passes run on the tcgen05 tensor cores.  Gate kinds, chunk tails,
    a single token, zero initial state without a final-state gradient."""
    _case(2, T, 40, 128, 128, torch.bfloat16, gate=gate, s0=s0, final=final, seed=120 + T)


def test_backward_tensor_core_passes_exact_path():
    """The exact pairwise path of the preparation (gates of exp(-20)) feeding the tensor-core passes."""
    dev = cuda_or_skip()
    B, T, H, d = 2, 150, 40, 128
    x = make_prefill_inputs(B, T, H, d, d, torch.bfloat16, 0.1, seed=131)
    g = x["g"].float()
    g[:, 64:128, :5, :8] = -20.0
    x["g"] = g.to(torch.bfloat16)
    d_o, d_s = make_cotangents(B, T, H, d, d, torch.bfloat16, seed=132)
    to = lambda t: t.to(dev)
    got = kda_backward(*(to(x[n]) for n in ("q", "k", "v", "g", "beta")), to(d_o), None, to(x["initial_state"]),
                       to(d_s))
    torch.cuda.synchronize()
    ref = oracle.kda_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], d ** -0.5, x["initial_state"], d_o, d_s)
    for name in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        assert rel_err(got[name], ref[name]) < TOL[torch.bfloat16], name


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_backward_empty_sequence(dtype):
    """T = 0: the token gradients are empty and dL/dS_0 = dL/dS_T (zeros
    when no final-state gradient is given)."""
    dev = cuda_or_skip()
    B, T, H, d = 2, 0, 2, 128
    x = make_prefill_inputs(B, T, H, d, d, dtype, 0.1, seed=171, device=dev)
    d_o, d_s = make_cotangents(B, T, H, d, d, dtype, seed=172, device=dev)
    args = (x["q"], x["k"], x["v"], x["g"], x["beta"], d_o, None, x["initial_state"])
    got = kda_backward(*args, d_s)
    torch.cuda.synchronize()
    for name in ("dq", "dk", "dv", "dg", "dbeta"):
        assert got[name].numel() == 0, name
    assert torch.equal(got["dS0"], d_s)
    got = kda_backward(*args, None)
    torch.cuda.synchronize()
    assert torch.count_nonzero(got["dS0"]) == 0
