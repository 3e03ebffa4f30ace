"""Scalar-gate forms through the same kernels: Gated DeltaNet (one log-gate per
token and head) and DeltaNet (no forget gate), against the fp64 oracle with
the gate broadcast over the key channels (the oracle's GDN and DeltaNet
reductions are pinned in tests/test_oracle_pins.py)."""
import pytest
import torch

import oracle
from gated_delta_rule_67_b200 import kda_chunk_fwd, kda_recurrent_step
from gated_delta_rule_67_b200.workloads import make_decode_inputs, make_head_gates, make_prefill_inputs
from tests.parity import TOL, cuda_or_skip, rel_err

pytestmark = pytest.mark.gpu
NAMES = ("q", "k", "v", "beta")


def _oracle_g(x, kind, gh):
    """The gate as the oracle reads it: per channel, broadcast from per head, or zero."""
    if kind == "head":
        return gh.unsqueeze(-1).expand_as(x["q"]).contiguous()
    return torch.zeros_like(x["q"])


def _prefill_case(kind, B, T, H, d, dtype, s0, seed):
    dev = cuda_or_skip()
    x = make_prefill_inputs(B, T, H, d, d, dtype, s0, seed=seed, device="cpu")
    gh = make_head_gates((B, T, H), 1, dtype, seed=seed + 500) if kind == "head" else None
    s0t = None if x["initial_state"] is None else x["initial_state"].to(dev)
    o, sT = kda_chunk_fwd(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), None if gh is None else gh.to(dev),
                          x["beta"].to(dev), d ** -0.5, s0t)
    torch.cuda.synchronize()
    ref_o, ref_s = oracle.kda_forward(x["q"], x["k"], x["v"], _oracle_g(x, kind, gh), x["beta"], d ** -0.5,
                                      x["initial_state"])
    assert rel_err(o, ref_o) < TOL[dtype]
    assert rel_err(sT, ref_s) < TOL[dtype]


@pytest.mark.parametrize("kind", ["head", "none"])
@pytest.mark.parametrize("B,T,H,s0", [(1, 64, 2, 0.1), (2, 200, 3, 0.0), (1, 1, 1, 0.1), (1, 64 * 13 + 5, 2, 0.1)])
def test_bf16_prefill_scalar_gates(kind, B, T, H, s0):
    """One chunk, ragged tails, a single token, and a few chains over many
    chunks (the chunk-parallel scan)."""
    _prefill_case(kind, B, T, H, 128, torch.bfloat16, s0, seed=60 + T)


@pytest.mark.parametrize("kind", ["head", "none"])
def test_bf16_prefill_scalar_gates_bench_shape(kind):
    """B=1, H=16, T=4096, d=128 with a random initial state."""
    _prefill_case(kind, 1, 4096, 16, 128, torch.bfloat16, 0.1, seed=61)


@pytest.mark.parametrize("kind", ["head", "none"])
@pytest.mark.parametrize("d", [64, 128])
def test_f32_prefill_scalar_gates(kind, d):
    _prefill_case(kind, 1, 256, 2, d, torch.float32, 0.1, seed=62)


@pytest.mark.parametrize("kind", ["head", "none"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_decode_scalar_gates(kind, dtype):
    dev = cuda_or_skip()
    steps, N, H, d = 6, 5, 3, 128
    x = make_decode_inputs(steps, N, H, d, d, dtype, 0.1, seed=63, device="cpu")
    gh = make_head_gates((steps, N, H), 0, dtype, seed=563) if kind == "head" else None
    g_or = gh.unsqueeze(-1).expand_as(x["q"]).contiguous() if kind == "head" else torch.zeros_like(x["q"])
    ref_o, ref_s = oracle.kda_decode(x["q"], x["k"], x["v"], g_or, x["beta"], d ** -0.5, x["state"])
    state = x["state"].to(dev)
    outs = [kda_recurrent_step(x["q"][t].to(dev), x["k"][t].to(dev), x["v"][t].to(dev),
                               None if gh is None else gh[t].to(dev), x["beta"][t].to(dev), state, d ** -0.5)
            for t in range(steps)]
    torch.cuda.synchronize()
    assert rel_err(torch.stack(outs), ref_o) < TOL[dtype]
    assert rel_err(state, ref_s) < TOL[dtype]


def test_head_gate_equals_broadcast_channel_gate():
    """Per-head gates give the same result as the per-channel path fed the
    broadcast gate (GPU vs GPU, bf16 prefill)."""
    dev = cuda_or_skip()
    x = make_prefill_inputs(1, 300, 2, 128, 128, torch.bfloat16, 0.1, seed=64, device=dev)
    gh = make_head_gates((1, 300, 2), 1, torch.bfloat16, seed=564, device=dev)
    o1, s1 = kda_chunk_fwd(x["q"], x["k"], x["v"], gh, x["beta"], None, x["initial_state"])
    o2, s2 = kda_chunk_fwd(x["q"], x["k"], x["v"], gh.unsqueeze(-1).expand_as(x["q"]).contiguous(), x["beta"], None,
                           x["initial_state"])
    torch.cuda.synchronize()
    assert rel_err(o1, o2.float()) < 1e-3
    assert rel_err(s1, s2) < 1e-3
