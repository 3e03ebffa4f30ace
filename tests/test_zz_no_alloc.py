"""The allocation-free prefill entry point (kda_chunk_fwd_noalloc).

Callers that cannot allocate device memory (a host program with no device
allocator of its own, or a plugin inside a framework that owns all device
memory) use the library's static device scratch instead of a workspace.
This checks, through the C ABI, that two calls in a row, the second smaller
than the first, give bit-identical results to the ordinary entry point with
its own workspace (the same deterministic kernels run on both paths, so a
stale scratch would show up as a difference), that the scratch's error word
reads clear after each call, that the second call also matches the fp64
oracle within the bf16 tolerance, and that a problem larger than the static
scratch is refused.  It is collected last on purpose.
"""
import pytest
import torch

import oracle
from gated_delta_rule_67_b200 import binding
from gated_delta_rule_67_b200.workloads import make_prefill_inputs
from tests.parity import TOL, cuda_or_skip, rel_err

pytestmark = pytest.mark.gpu
NAMES = ("q", "k", "v", "g", "beta")


def test_noalloc_matches_workspace_entry_point_twice():
    dev = cuda_or_skip()
    binding.load()
    for call, (B, T, H, seed) in enumerate([(2, 1000, 4, 61), (1, 333, 3, 62)]):
        x = make_prefill_inputs(B, T, H, 128, 128, torch.bfloat16, 0.1, seed=seed, device=dev)
        ins = [x[n] for n in NAMES]
        o_ref, s_ref = binding.kda_chunk_fwd(*ins, None, x["initial_state"])
        o_na, s_na = binding.kda_chunk_fwd_noalloc(*ins, None, x["initial_state"])
        assert binding.kda_chunk_fwd_noalloc_check(dev) == binding.KDA_OK, call
        torch.cuda.synchronize()
        assert torch.equal(o_na, o_ref), call
        assert torch.equal(s_na, s_ref), call
        if call == 1:
            ref_o, ref_s = oracle.kda_forward(*(x[n].cpu() for n in NAMES), 128 ** -0.5, x["initial_state"].cpu())
            assert rel_err(o_na, ref_o) < TOL[torch.bfloat16]
            assert rel_err(s_na, ref_s) < TOL[torch.bfloat16]


def test_noalloc_refuses_problems_beyond_the_scratch():
    dev = cuda_or_skip()
    binding.load()
    # 1 x 16 heads x ceil(4096/64)=64 chunks = 1024 chunk-heads: its workspace exceeds the 64 MiB
    # scratch, so the call is refused before any launch.
    x = make_prefill_inputs(1, 4096, 16, 128, 128, torch.bfloat16, 0.1, seed=63, device=dev)
    with pytest.raises(binding.KDAError) as e:
        binding.kda_chunk_fwd_noalloc(*(x[n] for n in NAMES), None, x["initial_state"])
    assert e.value.status == binding.KDA_ERR_UNSUPPORTED
