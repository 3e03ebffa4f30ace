"""Fused input preparation (kda_prep bits): raw projections in, the kernels
normalise q and k, apply log-sigmoid to g and sigmoid to beta; against the
fp64 oracle run on oracle.prepare_inputs of the same raw values."""
import pytest
import torch

import oracle
from gated_delta_rule_67_b200 import kda_chunk_fwd, kda_recurrent_step
from gated_delta_rule_67_b200.binding import (KDA_PREP_ALL, KDA_PREP_BETA_SIGMOID, KDA_PREP_GATE_LOGSIGMOID,
                                              KDA_PREP_L2NORM_QK)
from gated_delta_rule_67_b200.workloads import make_head_gates, make_raw_prefill_inputs
from tests.parity import TOL, cuda_or_skip, rel_err

pytestmark = pytest.mark.gpu


def _gate_for(kind, x, lead, seed, seq_axis=1):
    if kind == "channel":
        return x["g"]
    if kind == "head":
        return make_head_gates(lead, seq_axis, x["q"].dtype, seed=seed, raw=True)
    return None


def _oracle_g(kind, g, like):
    if kind == "channel":
        return g
    if kind == "head":
        return g.unsqueeze(-1).expand_as(like).contiguous()
    return torch.zeros_like(like)


def _check_prefill(x, kind, g, prep, dtype):
    dev = cuda_or_skip()
    d = x["q"].shape[-1]
    s0 = None if x["initial_state"] is None else x["initial_state"].to(dev)
    o, sT = kda_chunk_fwd(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), None if g is None else g.to(dev),
                          x["beta"].to(dev), d ** -0.5, s0, prep=prep)
    torch.cuda.synchronize()
    # the oracle prepares the broadcast gate exactly as the kernels prepare the per-head one
    q, k, gg, b = oracle.prepare_inputs(x["q"], x["k"], _oracle_g(kind, g, x["q"]), x["beta"], prep)
    if kind == "none":
        gg = 0.0 * gg
    ref_o, ref_s = oracle.kda_forward(q, k, x["v"], gg, b, d ** -0.5, x["initial_state"])
    assert rel_err(o, ref_o) < TOL[dtype]
    assert rel_err(sT, ref_s) < TOL[dtype]


@pytest.mark.parametrize("kind", ["channel", "head", "none"])
@pytest.mark.parametrize("B,T,H", [(1, 64, 2), (2, 200, 3), (1, 64 * 13 + 5, 2)])
def test_bf16_prefill_all_prep(kind, B, T, H):
    x = make_raw_prefill_inputs(B, T, H, 128, 128, torch.bfloat16, 0.1, seed=70 + T)
    _check_prefill(x, kind, _gate_for(kind, x, (B, T, H), 570 + T), KDA_PREP_ALL, torch.bfloat16)


@pytest.mark.parametrize("prep", [KDA_PREP_L2NORM_QK, KDA_PREP_GATE_LOGSIGMOID, KDA_PREP_BETA_SIGMOID],
                         ids=["l2norm", "gate", "beta"])
def test_bf16_prefill_single_bits(prep):
    """One preparation step at a time; the other inputs are given prepared."""
    from gated_delta_rule_67_b200.workloads import make_prefill_inputs
    x = make_prefill_inputs(1, 150, 2, 128, 128, torch.bfloat16, 0.1, seed=71)
    raw = make_raw_prefill_inputs(1, 150, 2, 128, 128, torch.bfloat16, 0.1, seed=72)
    if prep == KDA_PREP_L2NORM_QK:
        x["q"], x["k"] = raw["q"], raw["k"]
    elif prep == KDA_PREP_GATE_LOGSIGMOID:
        x["g"] = raw["g"]
    else:
        x["beta"] = raw["beta"]
    _check_prefill(x, "channel", x["g"], prep, torch.bfloat16)


def test_bf16_prefill_prep_bench_shape():
    x = make_raw_prefill_inputs(1, 4096, 16, 128, 128, torch.bfloat16, 0.1, seed=73)
    _check_prefill(x, "channel", x["g"], KDA_PREP_ALL, torch.bfloat16)


def test_bf16_prefill_prep_exact_path():
    """Raw gates of -30 in some chunks: log-sigmoid ~ -30 per token, so those
    chunks leave the factored form's range and take the exact per-pair path,
    where the unit-length factors are applied to the pair sums."""
    x = make_raw_prefill_inputs(1, 300, 2, 128, 128, torch.bfloat16, 0.1, seed=74)
    g = x["g"].float()
    g[:, 64:128, 0, :16] = -30.0
    g[:, 200:, 1, :] = -30.0
    x["g"] = g.to(torch.bfloat16)
    _check_prefill(x, "channel", x["g"], KDA_PREP_ALL, torch.bfloat16)


@pytest.mark.parametrize("kind", ["channel", "head"])
@pytest.mark.parametrize("d", [64, 128])
def test_f32_prefill_all_prep(kind, d):
    x = make_raw_prefill_inputs(1, 100, 2, d, d, torch.float32, 0.1, seed=75)
    _check_prefill(x, kind, _gate_for(kind, x, (1, 100, 2), 575), KDA_PREP_ALL, torch.float32)


@pytest.mark.parametrize("kind", ["channel", "head", "none"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_decode_all_prep(kind, dtype):
    dev = cuda_or_skip()
    steps, N, H, d = 5, 4, 3, 128
    r = make_raw_prefill_inputs(N, steps, H, d, d, dtype, 0.1, seed=76)  # [N, steps, H, d]: one sequence per row
    tr = lambda t: t.transpose(0, 1).contiguous()                        # -> [steps, N, H, ...]
    x = {n: tr(r[n]) for n in ("q", "k", "v", "g", "beta")}
    g = x["g"] if kind == "channel" else (make_head_gates((steps, N, H), 0, dtype, seed=576, raw=True)
                                          if kind == "head" else None)
    state0 = r["initial_state"]                                          # [N, H, d, d]
    q, k, gg, b = oracle.prepare_inputs(x["q"], x["k"], _oracle_g(kind, g, x["q"]), x["beta"], KDA_PREP_ALL)
    if kind == "none":
        gg = 0.0 * gg
    ref_o, ref_s = oracle.kda_decode(q, k, x["v"], gg, b, d ** -0.5, state0)
    state = state0.to(dev)
    outs = [kda_recurrent_step(x["q"][t].to(dev), x["k"][t].to(dev), x["v"][t].to(dev),
                               None if g is None else g[t].to(dev), x["beta"][t].to(dev), state, d ** -0.5,
                               prep=KDA_PREP_ALL) for t in range(steps)]
    torch.cuda.synchronize()
    assert rel_err(torch.stack(outs), ref_o) < TOL[dtype]
    assert rel_err(state, ref_s) < TOL[dtype]
