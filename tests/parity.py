"""Shared helpers of the GPU parity tests: the error metric and tolerances.

Error metric: max|x - x_ref| / max|x_ref| over the whole tensor, separately
for o and for the final state; tolerances 1e-4 for fp32 inputs and 1e-2 for
bf16 inputs (fp32 state and accumulation in both cases).
"""
import numpy as np
import torch

TOL = {torch.float32: 1e-4, torch.bfloat16: 1e-2}


def rel_err(x, ref) -> float:
    x = x.detach().double().cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x, np.float64)
    ref = ref.detach().double().cpu().numpy() if isinstance(ref, torch.Tensor) else np.asarray(ref, np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    assert np.isfinite(x).all(), "non-finite values in GPU result"
    denom = np.max(np.abs(ref))
    return float(np.max(np.abs(x - ref)) / (denom if denom > 0 else 1.0))


def cuda_or_skip():
    import pytest
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return torch.device("cuda:0")
