"""The prefill, decode and backward calls inside CUDA graphs: captured once,
replayed on new inputs copied into the captured buffers, bit-identical to
eager calls (the prefill and the backward chain their kernels with
programmatic dependent launch)."""
import pytest
import torch

from gated_delta_rule_67_b200 import kda_chunk_fwd, kda_chunk_fwd_workspace_size, kda_recurrent_step
from gated_delta_rule_67_b200.workloads import make_decode_inputs, make_prefill_inputs
from tests.parity import cuda_or_skip

pytestmark = pytest.mark.gpu
NAMES = ("q", "k", "v", "g", "beta")


@pytest.mark.parametrize("B,T,H", [(1, 4096, 16), (4, 512, 32)], ids=["scan", "many-chains"])
def test_prefill_graph_replay_matches_eager(B, T, H):
    dev = cuda_or_skip()
    xs = [make_prefill_inputs(B, T, H, 128, 128, torch.bfloat16, 0.1, seed=s, device=dev) for s in (120, 121)]
    ws = torch.empty(kda_chunk_fwd_workspace_size(B, T, H, 128, 128), dtype=torch.uint8, device=dev)
    buf = {n: xs[0][n].clone() for n in NAMES}
    s0 = xs[0]["initial_state"].clone()
    o = torch.empty_like(buf["v"])
    sT = torch.empty_like(s0)
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):  # warm-up (library setup) outside the capture
        kda_chunk_fwd(*(buf[n] for n in NAMES), None, s0, o=o, final_state=sT, workspace=ws)
    torch.cuda.current_stream(dev).wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        kda_chunk_fwd(*(buf[n] for n in NAMES), None, s0, o=o, final_state=sT, workspace=ws)
    for x in xs:
        for n in NAMES:
            buf[n].copy_(x[n])
        s0.copy_(x["initial_state"])
        graph.replay()
        ref_o, ref_s = kda_chunk_fwd(*(x[n] for n in NAMES), None, x["initial_state"])
        torch.cuda.synchronize()
        assert torch.equal(o, ref_o) and torch.equal(sT, ref_s)


def test_decode_graph_of_steps():
    """Eight decode steps captured as one graph, replayed twice; the state
    carried in place matches sixteen eager steps."""
    dev = cuda_or_skip()
    x = make_decode_inputs(16, 8, 4, 128, 128, torch.bfloat16, 0.1, seed=122, device=dev)
    st_eager = x["state"].clone()
    for t in range(16):
        kda_recurrent_step(*(x[n][t] for n in NAMES), st_eager)
    st = x["state"].clone()
    tok = {n: x[n][0].clone() for n in NAMES}
    o = torch.empty_like(x["v"][0])
    kda_recurrent_step(*(tok[n] for n in NAMES), st.clone(), o=o)  # library setup outside the capture
    torch.cuda.synchronize()
    seq = {n: x[n].clone() for n in NAMES}
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for t in range(8):
            kda_recurrent_step(*(seq[n][t] for n in NAMES), st, o=o)
    graph.replay()                         # steps 0-7
    for n in NAMES:
        seq[n][:8].copy_(x[n][8:16])
    graph.replay()                         # steps 8-15
    torch.cuda.synchronize()
    assert torch.equal(st, st_eager)


@pytest.mark.parametrize("dtype,prep", [(torch.bfloat16, 0), (torch.float32, 0), (torch.bfloat16, 7)],
                         ids=["bf16", "f32", "bf16-prep"])
def test_backward_graph_replay_matches_eager(dtype, prep):
    """kda_backward captured once (its four kernels chained by programmatic
    dependent launch; with preparation bits, six), replayed on new inputs:
    every gradient bit-identical to an eager call."""
    from gated_delta_rule_67_b200 import kda_backward
    from gated_delta_rule_67_b200.binding import load
    from gated_delta_rule_67_b200.workloads import make_cotangents
    dev = cuda_or_skip()
    B, T, H = 1, 300, 4
    xs = []
    for s in (123, 124):
        x = make_prefill_inputs(B, T, H, 128, 128, dtype, 0.1, seed=s, device=dev)
        x["d_o"], x["d_s"] = make_cotangents(B, T, H, 128, 128, dtype, seed=s + 10, device=dev)
        xs.append(x)
    keys = NAMES + ("d_o", "initial_state", "d_s")
    buf = {n: xs[0][n].clone() for n in keys}
    code = 1 if dtype == torch.bfloat16 else 0
    ws = torch.empty(int(load().kda_backward_ex_workspace_size(B, T, H, 128, 128, code, prep)), dtype=torch.uint8,
                     device=dev)

    def call(src):
        return kda_backward(*(src[n] for n in NAMES), src["d_o"], None, src["initial_state"], src["d_s"],
                            workspace=ws, prep=prep)

    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):  # warm-up (library setup) outside the capture
        call(buf)
    torch.cuda.current_stream(dev).wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        out = call(buf)
    for x in xs:
        for n in keys:
            buf[n].copy_(x[n])
        graph.replay()
        torch.cuda.synchronize()
        got = {n: t.clone() for n, t in out.items()}
        ref = call(x)
        torch.cuda.synchronize()
        for n in ref:
            assert torch.equal(got[n], ref[n]), n
