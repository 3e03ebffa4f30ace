"""fp32 prefill (kda_chunk_fwd, dtype fp32) against the fp64 oracle, through the C ABI."""
import pytest
import torch

import oracle
from gated_delta_rule_67_b200 import kda_chunk_fwd
from gated_delta_rule_67_b200.workloads import TINY_F32, make_config_inputs, make_prefill_inputs
from tests.parity import TOL, cuda_or_skip, rel_err

pytestmark = pytest.mark.gpu


def _check(x, dev, chunk=64, scale=None, tol=TOL[torch.float32]):
    dk = x["q"].shape[-1]
    scale = dk ** -0.5 if scale is None else scale
    ref_o, ref_s = oracle.kda_forward(x["q"], x["k"], x["v"], x["g"], x["beta"], scale, x["initial_state"])
    s0 = None if x["initial_state"] is None else x["initial_state"].to(dev)
    o, sT = kda_chunk_fwd(*(x[n].to(dev) for n in ("q", "k", "v", "g", "beta")), scale, s0, chunk=chunk)
    torch.cuda.synchronize()
    assert rel_err(o, ref_o) < tol
    assert rel_err(sT, ref_s) < tol
    return o, sT


def test_tiny_fp32_config():
    """B=1, H=2, T=256, d=64, chunk 64, zero initial state, seed 0."""
    dev = cuda_or_skip()
    _check(make_config_inputs(TINY_F32, device="cpu"), dev)


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_ragged_tail_and_random_state(dk, dv, chunk):
    dev = cuda_or_skip()
    x = make_prefill_inputs(2, 77, 3, dk, dv, torch.float32, 0.1, seed=31, device="cpu")
    _check(x, dev, chunk=chunk)


def test_in_place_state_and_split_calls():
    dev = cuda_or_skip()
    x = make_prefill_inputs(1, 150, 2, 128, 128, torch.float32, 0.1, seed=32, device=dev)
    o_full, s_full = kda_chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["initial_state"])
    state = x["initial_state"].clone()
    cut = 61
    part = lambda n, a, b: x[n][:, a:b].contiguous()
    o1, _ = kda_chunk_fwd(*(part(n, 0, cut) for n in ("q", "k", "v", "g", "beta")), None, state, final_state=state)
    o2, _ = kda_chunk_fwd(*(part(n, cut, 150) for n in ("q", "k", "v", "g", "beta")), None, state, final_state=state)
    torch.cuda.synchronize()
    assert rel_err(torch.cat([o1, o2], dim=1), o_full) < 1e-6
    assert rel_err(state, s_full) < 1e-6


def test_empty_sequence_copies_state():
    dev = cuda_or_skip()
    x = make_prefill_inputs(2, 0, 2, 64, 64, torch.float32, 0.1, seed=33, device=dev)
    o, sT = kda_chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["initial_state"])
    torch.cuda.synchronize()
    assert o.shape == (2, 0, 2, 64)
    assert torch.equal(sT, x["initial_state"])
    o, sT = kda_chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, None)
    torch.cuda.synchronize()
    assert torch.count_nonzero(sT) == 0
