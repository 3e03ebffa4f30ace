"""Decode step (kda_recurrent_step) against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_67_b200 import kda_recurrent_step, kda_chunk_fwd
from gated_delta_rule_67_b200.workloads import DECODE_BF16, make_decode_inputs, make_prefill_inputs
from tests.parity import TOL, cuda_or_skip, rel_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
def test_decode_small(dtype, dk, dv):
    dev = cuda_or_skip()
    steps, N, H = 6, 5, 3
    x = make_decode_inputs(steps, N, H, dk, dv, dtype, 0.1, seed=21, device="cpu")
    scale = dk ** -0.5
    ref_o, ref_s = oracle.kda_decode(x["q"], x["k"], x["v"], x["g"], x["beta"], scale, x["state"])
    state = x["state"].to(dev)
    outs = []
    for t in range(steps):
        outs.append(kda_recurrent_step(*(x[n][t].to(dev) for n in ("q", "k", "v", "g", "beta")), state, scale))
    o = torch.stack(outs)
    torch.cuda.synchronize()
    assert rel_err(o, ref_o) < TOL[dtype]
    assert rel_err(state, ref_s) < TOL[dtype]


def test_decode_full_shape_sampled_heads():
    """256 sequences x 32 heads, d=128, 1000 consecutive steps in place; the
    oracle follows a sample of (sequence, head) pairs through all steps, and o
    is compared at steps 1, 10, 100 and 1000."""
    dev = cuda_or_skip()
    c = DECODE_BF16
    x = make_decode_inputs(c.steps, c.N, c.H, c.dk, c.dv, c.torch_dtype, c.s0_std, c.seed, device=dev)
    state = x["state"].clone()
    check = {0, 9, 99, c.steps - 1}
    kept = {}
    for t in range(c.steps):
        o = kda_recurrent_step(x["q"][t], x["k"][t], x["v"][t], x["g"][t], x["beta"][t], state, c.scale)
        if t in check:
            kept[t] = o.clone()
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    pairs = [(0, 0), (c.N - 1, c.H - 1)] + [tuple(p) for p in zip(rng.integers(0, c.N, 6), rng.integers(0, c.H, 6))]
    for n, h in pairs:
        sel = lambda a: a[:, n:n + 1, h:h + 1]
        ref_o, ref_s = oracle.kda_decode(sel(x["q"]), sel(x["k"]), sel(x["v"]), sel(x["g"]), sel(x["beta"]),
                                         c.scale, x["state"][n:n + 1, h:h + 1])
        for t in check:
            assert rel_err(kept[t][n, h], ref_o[t, 0, 0]) < TOL[torch.bfloat16], (n, h, t)
        assert rel_err(state[n, h], ref_s[0, 0]) < TOL[torch.bfloat16], (n, h)


def test_decode_steps_equal_prefill():
    """T single-token steps carry the same state as one prefill over T tokens (fp32)."""
    dev = cuda_or_skip()
    B, T, H, d = 2, 40, 3, 128
    x = make_prefill_inputs(B, T, H, d, d, torch.float32, 0.1, seed=22, device=dev)
    o_p, s_p = kda_chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["initial_state"])
    state = x["initial_state"].clone()
    outs = [kda_recurrent_step(x["q"][:, t].contiguous(), x["k"][:, t].contiguous(), x["v"][:, t].contiguous(),
                               x["g"][:, t].contiguous(), x["beta"][:, t].contiguous(), state) for t in range(T)]
    o_d = torch.stack(outs, dim=1)
    torch.cuda.synchronize()
    assert rel_err(o_d, o_p) < 1e-5
    assert rel_err(state, s_p) < 1e-5


def test_decode_extreme_gates():
    """Gates of exp(-20) in some channels and exactly 1 in others stay finite and match."""
    dev = cuda_or_skip()
    steps, N, H, d = 4, 3, 2, 128
    x = make_decode_inputs(steps, N, H, d, d, torch.bfloat16, 0.1, seed=23, device="cpu")
    g = x["g"].float()
    g[..., : d // 2] = -20.0
    g[..., d // 2:] = 0.0
    x["g"] = g.to(torch.bfloat16)
    ref_o, ref_s = oracle.kda_decode(x["q"], x["k"], x["v"], x["g"], x["beta"], d ** -0.5, x["state"])
    state = x["state"].to(dev)
    o = torch.stack([kda_recurrent_step(*(x[n][t].to(dev) for n in ("q", "k", "v", "g", "beta")), state)
                     for t in range(steps)])
    torch.cuda.synchronize()
    assert rel_err(o, ref_o) < TOL[torch.bfloat16]
    assert rel_err(state, ref_s) < TOL[torch.bfloat16]
