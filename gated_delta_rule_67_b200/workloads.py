"""Seeded synthetic KDA workloads: the configuration table and input generators.

This module draws inputs only; it holds none of the operator's arithmetic, so
both the CUDA path and the fp64 oracle may consume what it produces.

Value recipe (identical for every configuration; the KimiLinear pages print
no dataset for the operator, so seeded synthetic tensors of the stated shapes
stand in for real activations):
  q, k   ~ N(0, 1) per element, then L2-normalised over the key channels of
           each token (in fp32), then cast to the configuration dtype;
  v      ~ N(0, 1);
  beta   = sigmoid(N(0, 1)), one scalar per (token, head);
  g      = logsigmoid(N(3, 1)) per key channel (log of the forget gate, so
           the gate exp(g) lies in (0, 1));
  S0     = zeros, or N(0, 0.1^2) per element (fp32) for the configurations
           with a random initial state.
Draw order: q, k, v, beta, g, then S0, each tensor drawn slab by slab along
the sequence axis from one generator seeded with the configuration's seed.
Low-precision tensors are produced by round-to-nearest-even from fp32.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch
import torch.nn.functional as F


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    chunk: int
    dtype: str          # "f32" or "bf16": dtype of q, k, v, g, beta and o
    s0_std: float       # 0.0 => zero initial state
    seed: int
    notes: str = ""

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.dk)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    N: int
    H: int
    dk: int
    dv: int
    steps: int
    dtype: str
    s0_std: float
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.dk)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


# The five workloads of the operator, named by what they are.
TINY_F32 = PrefillConfig("tiny_fp32_B1_H2_T256_d64", 1, 2, 256, 64, 64, 64, "f32", 0.0, 0)
PREFILL_BF16 = PrefillConfig("prefill_bf16_B1_H16_T4096_d128", 1, 16, 4096, 128, 128, 64, "bf16", 0.1, 1)
TRAIN_BF16 = PrefillConfig("train_bf16_B8_H32_T8192_d128", 8, 32, 8192, 128, 128, 64, "bf16", 0.1, 2)
LONG_BF16 = PrefillConfig("long_bf16_B1_H32_T1048576_d128", 1, 32, 1 << 20, 128, 128, 64, "bf16", 0.1, 3)
DECODE_BF16 = DecodeConfig("decode_bf16_N256_H32_d128_1000steps", 256, 32, 128, 128, 1000, "bf16", 0.1, 4)

# The first 65,536 tokens of the long-context workload (same seed, same
# recipe): the same chunk-parallel scan structure (3 groups per chain) at a
# size whose DRAM traffic a profiler can capture; per-call traffic scales with T.
LONG_PREFIX_BF16 = PrefillConfig("long_prefix_bf16_B1_H32_T65536_d128", 1, 32, 1 << 16, 128, 128, 64, "bf16", 0.1, 3)

PREFILL_CONFIGS = {c.name: c for c in (TINY_F32, PREFILL_BF16, TRAIN_BF16, LONG_BF16, LONG_PREFIX_BF16)}

_SLAB_ELEMS = 1 << 27  # fp32 elements drawn per slab (512 MB), bounds temporaries


def _gen(seed: int, device) -> torch.Generator:
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return gen


def _slabs(n_rows: int, row_elems: int):
    rows = max(1, _SLAB_ELEMS // max(1, row_elems))
    for r0 in range(0, n_rows, rows):
        yield r0, min(n_rows, r0 + rows)


def _draw(kind: str, shape, seq_axis: int, dtype, gen, device) -> torch.Tensor:
    """Draw one tensor of the recipe, slab by slab along ``seq_axis``."""
    out = torch.empty(shape, dtype=dtype, device=device)
    n = shape[seq_axis]
    row = math.prod(shape) // max(1, n)
    for r0, r1 in _slabs(n, row):
        sshape = list(shape)
        sshape[seq_axis] = r1 - r0
        x = torch.randn(sshape, generator=gen, device=device, dtype=torch.float32)
        if kind == "unit":
            x = x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)
        elif kind == "beta":
            x = torch.sigmoid(x)
        elif kind == "gate":
            x = F.logsigmoid(x + 3.0)
        elif kind == "gate_raw":
            x = x + 3.0
        out.narrow(seq_axis, r0, r1 - r0).copy_(x.to(dtype))
    return out


def make_prefill_inputs(B, T, H, dk, dv, dtype=torch.bfloat16, s0_std=0.1, seed=0, device="cpu"):
    """Seeded prefill inputs: dict with q, k, v, g, beta, initial_state (or None)."""
    gen = _gen(seed, device)
    q = _draw("unit", (B, T, H, dk), 1, dtype, gen, device)
    k = _draw("unit", (B, T, H, dk), 1, dtype, gen, device)
    v = _draw("normal", (B, T, H, dv), 1, dtype, gen, device)
    beta = _draw("beta", (B, T, H), 1, dtype, gen, device)
    g = _draw("gate", (B, T, H, dk), 1, dtype, gen, device)
    s0 = None
    if s0_std > 0:
        s0 = torch.randn((B, H, dk, dv), generator=gen, device=device, dtype=torch.float32) * s0_std
    return dict(q=q, k=k, v=v, g=g, beta=beta, initial_state=s0)


def make_config_inputs(cfg: PrefillConfig, device="cpu", T=None, B=None, H=None):
    """Inputs for a named configuration (optionally with a reduced T/B/H)."""
    return make_prefill_inputs(B or cfg.B, T or cfg.T, H or cfg.H, cfg.dk, cfg.dv, cfg.torch_dtype,
                               cfg.s0_std, cfg.seed, device)


def make_decode_inputs(steps, N, H, dk, dv, dtype=torch.bfloat16, s0_std=0.1, seed=0, device="cpu"):
    """Seeded decode inputs: per-step q, k, v, g [steps,N,H,d], beta [steps,N,H], state [N,H,dk,dv]."""
    gen = _gen(seed, device)
    q = _draw("unit", (steps, N, H, dk), 0, dtype, gen, device)
    k = _draw("unit", (steps, N, H, dk), 0, dtype, gen, device)
    v = _draw("normal", (steps, N, H, dv), 0, dtype, gen, device)
    beta = _draw("beta", (steps, N, H), 0, dtype, gen, device)
    g = _draw("gate", (steps, N, H, dk), 0, dtype, gen, device)
    state = torch.randn((N, H, dk, dv), generator=gen, device=device, dtype=torch.float32) * s0_std
    return dict(q=q, k=k, v=v, g=g, beta=beta, state=state)


def make_head_gates(lead_shape, seq_axis, dtype=torch.bfloat16, seed=0, device="cpu", raw=False):
    """Seeded per-head log-gates for the Gated DeltaNet form: one
    logsigmoid(N(3, 1)) value per (token, head) (``raw``: the N(3, 1) value
    before its log-sigmoid), shape ``lead_shape`` (e.g. [B, T, H] or
    [steps, N, H]), drawn from its own generator."""
    return _draw("gate_raw" if raw else "gate", tuple(lead_shape), seq_axis, dtype, _gen(seed, device), device)


def make_raw_prefill_inputs(B, T, H, dk, dv, dtype=torch.bfloat16, s0_std=0.1, seed=0, device="cpu"):
    """Seeded raw projections for the fused input preparation: q, k, v ~ N(0, 1)
    (not normalised), beta ~ N(0, 1) before its sigmoid, g ~ N(3, 1) per key
    channel before its log-sigmoid (so prepared, they follow the same
    distributions as make_prefill_inputs)."""
    gen = _gen(seed, device)
    q = _draw("normal", (B, T, H, dk), 1, dtype, gen, device)
    k = _draw("normal", (B, T, H, dk), 1, dtype, gen, device)
    v = _draw("normal", (B, T, H, dv), 1, dtype, gen, device)
    beta = _draw("normal", (B, T, H), 1, dtype, gen, device)
    g = _draw("gate_raw", (B, T, H, dk), 1, dtype, gen, device)
    s0 = None
    if s0_std > 0:
        s0 = torch.randn((B, H, dk, dv), generator=gen, device=device, dtype=torch.float32) * s0_std
    return dict(q=q, k=k, v=v, g=g, beta=beta, initial_state=s0)


def make_cotangents(B, T, H, dk, dv, dtype=torch.bfloat16, seed=0, device="cpu", final_state=True):
    """Seeded upstream gradients for the backward pass: dL/do ~ N(0, 1)
    [B, T, H, dv] (dtype) and, if ``final_state``, dL/dS_T ~ N(0, 0.1^2)
    [B, H, dk, dv] fp32 (else None)."""
    gen = _gen(seed, device)
    d_o = _draw("normal", (B, T, H, dv), 1, dtype, gen, device)
    d_s = torch.randn((B, H, dk, dv), generator=gen, device=device, dtype=torch.float32) * 0.1 if final_state else None
    return d_o, d_s
