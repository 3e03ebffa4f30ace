"""The bounded-wait failure path on the device: a wait that can never be
satisfied gives up after a short limit, the host reads KDA_ERR_TIMEOUT, and
the context stays usable for a correct call afterwards."""
import pytest
import torch

import oracle
from gated_delta_rule_67_b200 import binding
from gated_delta_rule_67_b200.workloads import make_prefill_inputs
from tests.parity import TOL, cuda_or_skip, rel_err

pytestmark = pytest.mark.gpu


def test_unsatisfiable_wait_reports_timeout_and_context_survives():
    dev = cuda_or_skip()
    ws = torch.empty(256, dtype=torch.uint8, device=dev)
    assert binding.kda_wait_selftest(ws) == binding.KDA_ERR_TIMEOUT
    # the same workspace is cleared by the next real call, and results are valid
    x = make_prefill_inputs(1, 70, 2, 128, 128, torch.bfloat16, 0.1, seed=81, device="cpu")
    names = ("q", "k", "v", "g", "beta")
    need = binding.kda_chunk_fwd_workspace_size(1, 70, 2, 128, 128)
    big = torch.empty(need, dtype=torch.uint8, device=dev)
    o, sT = binding.kda_chunk_fwd(*(x[n].to(dev) for n in names), None, x["initial_state"].to(dev), workspace=big)
    assert binding.kda_chunk_fwd_check(big) == binding.KDA_OK
    ref_o, ref_s = oracle.kda_forward(*(x[n] for n in names), 128 ** -0.5, x["initial_state"])
    assert rel_err(o, ref_o) < TOL[torch.bfloat16] and rel_err(sT, ref_s) < TOL[torch.bfloat16]
