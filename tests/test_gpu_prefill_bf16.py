"""bf16 chunked prefill (tcgen05 path) against the fp64 oracle, through the C ABI."""
import pytest
import torch

import oracle
from gated_delta_rule_67_b200 import kda_chunk_fwd, kda_chunk_fwd_check, kda_chunk_fwd_workspace_size
from gated_delta_rule_67_b200.workloads import (LONG_BF16, PREFILL_BF16, TRAIN_BF16, make_config_inputs,
                                                make_prefill_inputs)
from tests.parity import TOL, cuda_or_skip, rel_err

pytestmark = pytest.mark.gpu
TOLB = TOL[torch.bfloat16]
NAMES = ("q", "k", "v", "g", "beta")


def _run(x, dev, scale=None, ws=None):
    d = x["q"].shape[-1]
    scale = d ** -0.5 if scale is None else scale
    s0 = None if x["initial_state"] is None else x["initial_state"].to(dev)
    o, sT = kda_chunk_fwd(*(x[n].to(dev) for n in NAMES), scale, s0, workspace=ws)
    torch.cuda.synchronize()
    return o, sT


def _oracle(x, scale=None):
    d = x["q"].shape[-1]
    scale = d ** -0.5 if scale is None else scale
    return oracle.kda_forward(*(x[n] for n in NAMES), scale, x["initial_state"])


@pytest.mark.parametrize("B,T,H,s0", [(1, 64, 1, 0.1), (1, 64, 2, 0.0), (2, 200, 3, 0.1), (1, 1, 2, 0.1),
                                      (1, 127, 2, 0.1), (3, 320, 2, 0.0)])
def test_small_shapes(B, T, H, s0):
    """One chunk, several chunks, a ragged tail, a single token, zero and random initial state."""
    dev = cuda_or_skip()
    x = make_prefill_inputs(B, T, H, 128, 128, torch.bfloat16, s0, seed=41 + T, device="cpu")
    o, sT = _run(x, dev)
    ref_o, ref_s = _oracle(x)
    assert rel_err(o, ref_o) < TOLB
    assert rel_err(sT, ref_s) < TOLB


def test_prefill_config_full():
    """B=1, H=16, T=4096, d=128, random initial state: every output against the oracle."""
    dev = cuda_or_skip()
    x = make_config_inputs(PREFILL_BF16, device="cpu")
    o, sT = _run(x, dev)
    ref_o, ref_s = _oracle(x)
    assert rel_err(o, ref_o) < TOLB
    assert rel_err(sT, ref_s) < TOLB


def _per_batch_against_oracle(cfg, zero_state=False):
    """One launch over the whole configuration, then every (sequence, head)
    chain against the oracle, one sequence (all heads) per oracle call."""
    dev = cuda_or_skip()
    x = make_config_inputs(cfg, device=dev)
    if zero_state:
        x["initial_state"] = None
    o, sT = _run(x, dev)
    worst_o = worst_s = 0.0
    for b in range(cfg.B):
        sel = {n: x[n][b:b + 1].cpu() for n in NAMES}
        sel["initial_state"] = None if x["initial_state"] is None else x["initial_state"][b:b + 1].cpu()
        ref_o, ref_s = _oracle(sel)
        eo, es = rel_err(o[b:b + 1], ref_o), rel_err(sT[b:b + 1], ref_s)
        assert eo < TOLB and es < TOLB, (b, eo, es)
        worst_o, worst_s = max(worst_o, eo), max(worst_s, es)
    return worst_o, worst_s


def test_train_config_every_chain():
    """B=8, H=32, T=8192, random initial state, in one launch: all 256 chains
    (o and final state) against the oracle."""
    _per_batch_against_oracle(TRAIN_BF16)


def test_train_config_every_chain_zero_state():
    _per_batch_against_oracle(TRAIN_BF16, zero_state=True)


def test_long_context_eight_heads():
    """T = 1,048,576 (16384 chunks carried in one chain per head, through the
    chunk-parallel scan) in one launch; the oracle follows 8 of the 32 heads
    end to end, the first and the last among them, two heads per call."""
    dev = cuda_or_skip()
    x = make_config_inputs(LONG_BF16, device=dev)
    o, sT = _run(x, dev)
    for h0 in (0, 9, 20, 30):
        sl = slice(h0, h0 + 2)
        sel = {n: x[n][:, :, sl].contiguous().cpu() for n in NAMES}
        sel["initial_state"] = x["initial_state"][:, sl].cpu()
        ref_o, ref_s = _oracle(sel)
        assert rel_err(o[:, :, sl], ref_o) < TOLB, h0
        assert rel_err(sT[:, sl], ref_s) < TOLB, h0
        del sel, ref_o, ref_s


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("B,T,H,s0", [(1, 1, 2, 0.1), (2, 200, 3, 0.1), (1, 127, 2, 0.0), (1, 64 * 13 + 5, 2, 0.1)])
def test_bf16_head_dims_64(dk, dv, B, T, H, s0):
    """d_k, d_v in {64, 128} on the tcgen05 path (64 channels zero-padded to
    128 inside the kernels): a single token, ragged tails, zero and random
    initial state, and a chunk-parallel scan shape (13 chunks + 5 tokens)."""
    dev = cuda_or_skip()
    x = make_prefill_inputs(B, T, H, dk, dv, torch.bfloat16, s0, seed=90 + T + dk + dv, device="cpu")
    o, sT = _run(x, dev)
    ref_o, ref_s = _oracle(x)
    assert rel_err(o, ref_o) < TOLB
    assert rel_err(sT, ref_s) < TOLB


def test_bf16_head_dim_64_extreme_gates_in_place():
    """d = 64 with exact-path chunks (gates of exp(-20)), zero-gate channels,
    a scan shape and the final state written over the initial state."""
    dev = cuda_or_skip()
    B, T, H, d = 1, 64 * 30, 2, 64
    x = make_prefill_inputs(B, T, H, d, d, torch.bfloat16, 0.1, seed=93, device="cpu")
    g = x["g"].float()
    g[:, 600:700, 0, :8] = -20.0
    g[:, :, 1, 40:] = 0.0
    x["g"] = g.to(torch.bfloat16)
    ref_o, ref_s = _oracle(x)
    state = x["initial_state"].to(dev)
    o, _ = kda_chunk_fwd(*(x[n].to(dev) for n in NAMES), None, state, final_state=state)
    torch.cuda.synchronize()
    assert rel_err(o, ref_o) < TOLB
    assert rel_err(state, ref_s) < TOLB


def test_split_calls_and_in_place_state():
    """Cutting the sequence (at a chunk boundary and inside a chunk) and carrying
    final_state -> initial_state in place matches one call."""
    dev = cuda_or_skip()
    x = make_prefill_inputs(2, 300, 2, 128, 128, torch.bfloat16, 0.1, seed=44, device=dev)
    o_full, s_full = kda_chunk_fwd(*(x[n] for n in NAMES), None, x["initial_state"])
    state = x["initial_state"].clone()
    outs = []
    for a, b in ((0, 64), (64, 101), (101, 300)):
        part = [x[n][:, a:b].contiguous() for n in NAMES]
        oo, _ = kda_chunk_fwd(*part, None, state, final_state=state)
        outs.append(oo)
    torch.cuda.synchronize()
    ref_o, ref_s = _oracle({n: x[n] for n in NAMES} | {"initial_state": x["initial_state"]})
    assert rel_err(torch.cat(outs, dim=1), ref_o) < TOLB
    assert rel_err(state, ref_s) < TOLB
    assert rel_err(o_full, ref_o) < TOLB


def test_matches_decode_steps():
    """A prefill over T tokens equals T single-token decode steps (GPU vs GPU)."""
    from gated_delta_rule_67_b200 import kda_recurrent_step
    dev = cuda_or_skip()
    x = make_prefill_inputs(2, 96, 4, 128, 128, torch.bfloat16, 0.1, seed=45, device=dev)
    o_p, s_p = kda_chunk_fwd(*(x[n] for n in NAMES), None, x["initial_state"])
    state = x["initial_state"].clone()
    o_d = torch.stack([kda_recurrent_step(*(x[n][:, t].contiguous() for n in NAMES), state)
                       for t in range(96)], dim=1)
    torch.cuda.synchronize()
    assert rel_err(o_p, o_d) < TOLB
    assert rel_err(s_p, state) < TOLB


def test_workspace_reuse_and_check():
    """A caller-provided workspace can be reused; the on-device error word stays clear."""
    dev = cuda_or_skip()
    x = make_prefill_inputs(1, 256, 2, 128, 128, torch.bfloat16, 0.1, seed=46, device="cpu")
    need = kda_chunk_fwd_workspace_size(1, 256, 2, 128, 128)
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    ws.fill_(0xAB)
    o1, s1 = _run(x, dev, ws=ws)
    assert kda_chunk_fwd_check(ws) == 0
    o2, s2 = _run(x, dev, ws=ws)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)  # deterministic
    ref_o, ref_s = _oracle(x)
    assert rel_err(o1, ref_o) < TOLB and rel_err(s1, ref_s) < TOLB


@pytest.mark.parametrize("pattern", ["half_channels", "some_chunks", "all"])
def test_extreme_gates(pattern):
    """Gates of exp(-20) per token (cumulative decay far below e^-64 within a
    chunk) next to gates of exactly 1: the chunks that need it take the exact
    per-pair path; results stay finite and match the oracle."""
    dev = cuda_or_skip()
    B, T, H, d = 1, 300, 2, 128
    x = make_prefill_inputs(B, T, H, d, d, torch.bfloat16, 0.1, seed=47, device="cpu")
    g = x["g"].float()
    if pattern == "half_channels":
        g[..., : d // 2] = -20.0
        g[..., d // 2:] = 0.0
    elif pattern == "some_chunks":
        g[:, 64:128, :, :5] = -20.0   # chunk 1 only, a few channels
        g[:, 200:260, 1, :] = -3.0    # chunks 3-4 of head 1: -3 per token crosses -64 inside the chunk
    else:
        g[:] = -20.0
    x["g"] = g.to(torch.bfloat16)
    o, sT = _run(x, dev)
    ref_o, ref_s = _oracle(x)
    assert rel_err(o, ref_o) < TOLB
    assert rel_err(sT, ref_s) < TOLB


def test_gate_span_just_inside_fast_path():
    """Per-token log-gate of -0.95: the chunk's cumulative decay (-60.8) stays
    inside the factored form's safe range, with factors up to e^30 each way."""
    dev = cuda_or_skip()
    x = make_prefill_inputs(1, 256, 2, 128, 128, torch.bfloat16, 0.1, seed=48, device="cpu")
    x["g"] = torch.full_like(x["g"], -0.95)
    o, sT = _run(x, dev)
    ref_o, ref_s = _oracle(x)
    assert rel_err(o, ref_o) < TOLB
    assert rel_err(sT, ref_s) < TOLB


@pytest.mark.parametrize("B,T,H", [(1, 64 * 13 + 5, 2), (1, 64 * 40, 1), (2, 64 * 24 + 63, 3)])
def test_chunk_parallel_scan_shapes(B, T, H):
    """Few chains over many chunks take the chunk-parallel scan (groups of
    chunks, per-group transition and offset, fp32 combination, outputs per
    group); a ragged tail and a random initial state, against the oracle."""
    dev = cuda_or_skip()
    x = make_prefill_inputs(B, T, H, 128, 128, torch.bfloat16, 0.1, seed=50 + T, device="cpu")
    o, sT = _run(x, dev)
    ref_o, ref_s = _oracle(x)
    assert rel_err(o, ref_o) < TOLB
    assert rel_err(sT, ref_s) < TOLB


def test_scan_with_extreme_gates_and_in_place_state():
    """The scan path with exact-path chunks inside its groups, zero gate (no
    decay) channels, and the final state written over the initial state."""
    dev = cuda_or_skip()
    B, T, H = 1, 64 * 30, 2
    x = make_prefill_inputs(B, T, H, 128, 128, torch.bfloat16, 0.1, seed=77, device="cpu")
    g = x["g"].float()
    g[:, 600:700, 0, :8] = -20.0
    g[:, :, 1, 100:] = 0.0
    x["g"] = g.to(torch.bfloat16)
    ref_o, ref_s = _oracle(x)
    state = x["initial_state"].to(dev)
    o, _ = kda_chunk_fwd(*(x[n].to(dev) for n in NAMES), None, state, final_state=state)
    torch.cuda.synchronize()
    assert rel_err(o, ref_o) < TOLB
    assert rel_err(state, ref_s) < TOLB


@pytest.mark.parametrize("d,in_place", [(128, False), (64, True)])
def test_long_chains_light_offset_passes(d, in_place):
    """Few chains of many chunks (8 heads x 2600 chunks and a ragged tail):
    the scan's offset and transition passes run two per SM on the light
    instance of the state pass, with more groups; against the oracle (with
    d = 64 and the final state written over the initial state as well)."""
    dev = cuda_or_skip()
    B, T, H = 1, 64 * 2600 + 17, 8
    x = make_prefill_inputs(B, T, H, d, d, torch.bfloat16, 0.1, seed=150 + d, device="cpu")
    ref_o, ref_s = _oracle(x)
    state = x["initial_state"].to(dev)
    o, sT = kda_chunk_fwd(*(x[n].to(dev) for n in NAMES), None, state, final_state=state if in_place else None)
    torch.cuda.synchronize()
    assert rel_err(o, ref_o) < TOLB
    assert rel_err(state if in_place else sT, ref_s) < TOLB


@pytest.mark.parametrize("B,T", [(2, 0), (0, 64)], ids=["no-tokens", "no-sequences"])
def test_empty_inputs(B, T):
    """Nothing to run: the call succeeds without a workspace, o is empty, and
    the final state is the initial state (or zeros without one)."""
    dev = cuda_or_skip()
    H, d = 2, 128
    x = make_prefill_inputs(B, T, H, d, d, torch.bfloat16, 0.1, seed=170, device=dev)
    o, sT = kda_chunk_fwd(*(x[n] for n in NAMES), None, x["initial_state"])
    torch.cuda.synchronize()
    assert o.shape == (B, T, H, d)
    assert torch.equal(sT, x["initial_state"])
    o, sT = kda_chunk_fwd(*(x[n] for n in NAMES), None, None)
    torch.cuda.synchronize()
    assert sT.shape == (B, H, d, d) and torch.count_nonzero(sT) == 0


@pytest.mark.parametrize("B,T,H", [(1, 200, 2), (1, 64 * 13 + 5, 2)], ids=["one-pass", "scan"])
def test_no_writes_pure_decay(B, T, H):
    """beta = 0: nothing is written, the state only decays channel by channel,
    S_T = Diag(exp(sum_t g_t)) S0 and o_t = scale (Diag(exp(sum_{s<=t} g_s)) S0)^T q_t;
    against the oracle and against that closed form for the final state."""
    dev = cuda_or_skip()
    x = make_prefill_inputs(B, T, H, 128, 128, torch.bfloat16, 0.1, seed=173 + T, device="cpu")
    x["beta"] = torch.zeros_like(x["beta"])
    o, sT = _run(x, dev)
    ref_o, ref_s = _oracle(x)
    assert rel_err(o, ref_o) < TOLB
    assert rel_err(sT, ref_s) < TOLB
    decay = torch.exp(x["g"].double().sum(dim=1))             # [B, H, dk]
    closed = decay.unsqueeze(-1) * x["initial_state"].double()  # Diag(alpha) S0, per key channel
    assert rel_err(sT, closed) < TOLB
