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
    # the cut at token 61 moves every later chunk boundary, so the two runs round differently (fp32)
    assert rel_err(torch.cat([o1, o2], dim=1), o_full) < 1e-5
    assert rel_err(state, s_full) < 1e-5


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


@pytest.mark.parametrize("dk", [64, 128])
def test_chunk_size_changes_the_arithmetic_not_the_result(dk):
    """The fp32 path evaluates the chunk form with the caller's chunk size:
    C in {16, 32, 64} must agree with one another far inside the tolerance,
    each must meet the oracle, and they must not be bit-identical (the chunk
    size really selects a different evaluation)."""
    dev = cuda_or_skip()
    x = make_prefill_inputs(1, 200, 2, dk, dk, torch.float32, 0.1, seed=34 + dk, device="cpu")
    res = {c: _check(x, dev, chunk=c) for c in (16, 32, 64)}
    for c in (16, 32):
        assert rel_err(res[c][0], res[64][0]) < 1e-5 and rel_err(res[c][1], res[64][1]) < 1e-5
    assert not torch.equal(res[16][0], res[64][0])


@pytest.mark.parametrize("gate", ["head", "none"])
def test_scalar_gates_chunked(gate):
    dev = cuda_or_skip()
    x = make_prefill_inputs(1, 100, 2, 64, 64, torch.float32, 0.1, seed=36, device="cpu")
    if gate == "head":
        x["g"] = x["g"][..., 0].contiguous()
        ref = dict(x, g=x["g"].unsqueeze(-1).expand(-1, -1, -1, 64).contiguous())
    else:
        x["g"] = None
        ref = dict(x, g=torch.zeros(1, 100, 2, 64))
    ref_o, ref_s = oracle.kda_forward(ref["q"], ref["k"], ref["v"], ref["g"], ref["beta"], 64 ** -0.5,
                                      ref["initial_state"])
    for c in (16, 64):
        o, sT = kda_chunk_fwd(*(None if x[n] is None else x[n].to(dev) for n in ("q", "k", "v", "g", "beta")), None,
                              x["initial_state"].to(dev), chunk=c)
        torch.cuda.synchronize()
        assert rel_err(o, ref_o) < TOL[torch.float32] and rel_err(sT, ref_s) < TOL[torch.float32]
