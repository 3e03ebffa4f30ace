"""The C ABI on the host: the library loads, exports every declared symbol,
and rejects bad arguments before touching the GPU (no device needed)."""
import ctypes
import os
import re

import pytest

from gated_delta_rule_67_b200 import binding
from gated_delta_rule_67_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"KDA_API\s+[\w\s\*]+?\b(kda_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    assert declared_symbols() == sorted(binding.SIGNATURES)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for s in range(5):
        assert binding.status_string(s).startswith("KDA_")
    assert "UNKNOWN" in binding.status_string(99)
    assert binding.version() >= 100


def test_workspace_size_rejects_bad_args(lib):
    f = lib.kda_chunk_fwd_workspace_size
    assert f(1, 64, 1, 128, 128, 64, 9) == 0      # bad dtype
    assert f(-1, 64, 1, 128, 128, 64, 1) == 0     # bad B
    assert f(1, 64, 1, 96, 96, 64, 1) == 0        # unsupported d
    assert f(1, 64, 1, 64, 64, 64, 0) == 0        # fp32 path needs none
    # bf16 takes d in {64, 128} (64 channels zero-padded inside the kernels): the same workspace
    assert f(1, 64, 1, 64, 64, 64, 1) == f(1, 64, 1, 128, 128, 64, 1) > 0
    assert f(1, 64, 1, 64, 128, 64, 1) > 0


# Fake device addresses: validation must fail before any CUDA call is made.
A = 1 << 40


def _fwd(lib, q=A, k=A + (1 << 30), v=A + (2 << 30), g=A + (3 << 30), beta=A + (4 << 30), s0=None,
         o=A + (5 << 30), sT=None, B=1, T=64, H=1, dk=128, dv=128, chunk=64, dtype=1, ws=None, wsb=0, scale=1.0):
    return lib.kda_chunk_fwd(q, k, v, g, beta, scale, s0, o, sT, B, T, H, dk, dv, chunk, dtype, ws, wsb, None)


def test_chunk_fwd_rejects_null_and_misaligned(lib):
    assert _fwd(lib, q=None) == binding.KDA_ERR_INVALID_ARG
    assert _fwd(lib, o=None) == binding.KDA_ERR_INVALID_ARG
    assert _fwd(lib, k=A + 8) == binding.KDA_ERR_INVALID_ARG
    assert _fwd(lib, s0=A + (6 << 30) + 4) == binding.KDA_ERR_INVALID_ARG
    assert _fwd(lib, T=-1) == binding.KDA_ERR_INVALID_ARG
    assert _fwd(lib, H=0) == binding.KDA_ERR_INVALID_ARG
    assert _fwd(lib, dtype=5) == binding.KDA_ERR_INVALID_ARG
    assert _fwd(lib, scale=float("nan")) == binding.KDA_ERR_INVALID_ARG


def test_chunk_fwd_rejects_overlap(lib):
    assert _fwd(lib, o=A + 64) == binding.KDA_ERR_INVALID_ARG                 # o overlaps q
    assert _fwd(lib, sT=A + (2 << 30)) == binding.KDA_ERR_INVALID_ARG         # final state overlaps v


def test_chunk_fwd_unsupported_shapes(lib):
    assert _fwd(lib, dk=96, dv=96) == binding.KDA_ERR_UNSUPPORTED
    assert _fwd(lib, dtype=0, chunk=48, dk=64, dv=64) == binding.KDA_ERR_UNSUPPORTED
    assert _fwd(lib, dtype=0, dk=64, dv=32) == binding.KDA_ERR_UNSUPPORTED


def test_chunk_fwd_workspace_checked(lib):
    need = lib.kda_chunk_fwd_workspace_size(1, 64, 1, 128, 128, 64, 1)
    if need == 0:
        pytest.skip("bf16 path needs no workspace")
    assert _fwd(lib, ws=None, wsb=0) == binding.KDA_ERR_INVALID_ARG
    assert _fwd(lib, ws=A + (7 << 30), wsb=need - 1) == binding.KDA_ERR_INVALID_ARG
    assert _fwd(lib, ws=A + (7 << 30) + 16, wsb=need) == binding.KDA_ERR_INVALID_ARG  # not 256-aligned


def test_recurrent_step_validation(lib):
    f = lib.kda_recurrent_step
    args = [A, A + (1 << 30), A + (2 << 30), A + (3 << 30), A + (4 << 30), 1.0, A + (5 << 30), A + (6 << 30)]
    assert f(*args, 0, 1, 128, 128, 1, None) == binding.KDA_OK          # N = 0: nothing to do
    bad = list(args)
    bad[0] = None
    assert f(*bad, 4, 1, 128, 128, 1, None) == binding.KDA_ERR_INVALID_ARG
    bad = list(args)
    bad[7] = A + 32                                                        # o overlaps q
    assert f(*bad, 4, 1, 128, 128, 1, None) == binding.KDA_ERR_INVALID_ARG
    assert f(*args, 4, 1, 96, 128, 1, None) == binding.KDA_ERR_UNSUPPORTED
    assert f(*args, 4, 1, 128, 128, 3, None) == binding.KDA_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 4, 1, 64)
    with pytest.raises(ValueError, match="CUDA"):
        binding.kda_chunk_fwd(x, x, x, x, torch.zeros(1, 4, 1))


def test_wait_selftest_validation(lib):
    assert lib.kda_wait_selftest(None, 256, None) == binding.KDA_ERR_INVALID_ARG
    assert lib.kda_wait_selftest(A, 128, None) == binding.KDA_ERR_INVALID_ARG
    assert lib.kda_wait_selftest(A + 16, 256, None) == binding.KDA_ERR_INVALID_ARG


def test_launch_count(lib):
    f = lib.kda_chunk_fwd_launch_count
    assert f(1, 64, 1, 128, 128, 64, 1) == 2        # prep + one state pass
    assert f(1, 4096, 16, 128, 128, 64, 1) == 4     # few chains, many chunks: chunk-parallel scan
    assert f(8, 8192, 32, 128, 128, 64, 1) == 2     # many chains: one state pass
    assert f(1, 1 << 20, 32, 128, 128, 64, 1) == 5  # long chains: group 0's outputs as a launch of their own
    assert f(1, 256, 2, 64, 64, 64, 0) == 1         # fp32 path
    assert f(0, 64, 1, 128, 128, 64, 1) == 0
    assert f(1, 64, 1, 96, 96, 64, 1) == -1
    assert f(1, 64, 1, 128, 128, 64, 7) == -1


def _fwd_gate(lib, gate, g=A + (3 << 30), dtype=1, prep=0, **kw):
    a = dict(q=A, k=A + (1 << 30), v=A + (2 << 30), beta=A + (4 << 30), o=A + (5 << 30), B=1, T=64, H=1, dk=128,
             dv=128, chunk=64)
    a.update(kw)
    return lib.kda_chunk_fwd_ex(a["q"], a["k"], a["v"], g, a["beta"], 1.0, None, a["o"], None, a["B"], a["T"],
                                a["H"], a["dk"], a["dv"], a["chunk"], dtype, gate, prep, None, 0, None)


def test_chunk_fwd_gate_validation(lib):
    assert _fwd_gate(lib, 3) == binding.KDA_ERR_INVALID_ARG                   # unknown gate
    assert _fwd_gate(lib, 0, prep=8) == binding.KDA_ERR_INVALID_ARG           # unknown prep bit
    assert _fwd_gate(lib, 0, g=None) == binding.KDA_ERR_INVALID_ARG           # per-channel gate needs g
    assert _fwd_gate(lib, 1, g=None) == binding.KDA_ERR_INVALID_ARG           # per-head gate needs g
    assert _fwd_gate(lib, 0, g=A + (3 << 30) + 2) == binding.KDA_ERR_INVALID_ARG   # [.., dk] needs 16-B alignment
    # per-head g only needs element alignment; the bf16 path then wants its workspace (none given)
    assert _fwd_gate(lib, 1, g=A + (3 << 30) + 2) == binding.KDA_ERR_INVALID_ARG
    assert _fwd_gate(lib, 2, g=A + (5 << 30)) == binding.KDA_ERR_INVALID_ARG  # g ignored; workspace missing
    assert _fwd_gate(lib, 1, g=A + (5 << 30) + 64) == binding.KDA_ERR_INVALID_ARG  # o overlaps the per-head g


def test_recurrent_step_gate_validation(lib):
    f = lib.kda_recurrent_step_ex
    args = [A, A + (1 << 30), A + (2 << 30)]
    rest = [A + (4 << 30), 1.0, A + (5 << 30), A + (6 << 30)]
    assert f(*args, None, *rest, 4, 1, 128, 128, 1, 3, 0, None) == binding.KDA_ERR_INVALID_ARG   # unknown gate
    assert f(*args, None, *rest, 4, 1, 128, 128, 1, 2, 9, None) == binding.KDA_ERR_INVALID_ARG   # unknown prep bit
    assert f(*args, None, *rest, 4, 1, 128, 128, 1, 1, 0, None) == binding.KDA_ERR_INVALID_ARG   # per-head needs g
    assert f(*args, None, *rest, 0, 1, 128, 128, 1, 2, 7, None) == binding.KDA_OK                # N = 0
    bad_o = list(rest)
    bad_o[3] = A + (3 << 30) + 8                                                              # o overlaps g [N,H]
    assert f(*args, A + (3 << 30), *bad_o, 4, 1, 128, 128, 1, 1, 0, None) == binding.KDA_ERR_INVALID_ARG


def test_backward_validation(lib):
    f = lib.kda_backward
    assert lib.kda_backward_workspace_size(1, 64, 1, 128, 128, 1) > 0
    assert lib.kda_backward_workspace_size(1, 64, 1, 96, 128, 1) == 0
    ins = [A, A + (1 << 30), A + (2 << 30), A + (3 << 30), A + (4 << 30)]   # q k v g beta
    grads = [A + (10 << 30), A + (11 << 30), A + (12 << 30), A + (13 << 30), A + (14 << 30)]

    def call(ins=ins, grads=grads, gate=0, dk=128, dv=128, ws=A + (20 << 30), wsb=1 << 40, grad_o=A + (5 << 30)):
        return f(*ins, 1.0, None, grad_o, None, *grads, None, 1, 64, 1, dk, dv, 1, gate, ws, wsb, None)

    assert call(gate=3) == binding.KDA_ERR_INVALID_ARG
    assert call(dk=96) == binding.KDA_ERR_UNSUPPORTED
    assert call(ws=None) == binding.KDA_ERR_INVALID_ARG
    assert call(wsb=16) == binding.KDA_ERR_INVALID_ARG
    one = lib.kda_backward_workspace_size(1, 64, 1, 128, 128, 1)
    assert lib.kda_backward_ex_workspace_size(1, 64, 1, 128, 128, 1, 0) == one
    assert lib.kda_backward_ex_workspace_size(1, 64, 1, 128, 128, 1, 7) > one
    assert lib.kda_backward_ex_workspace_size(1, 64, 1, 128, 128, 1, 8) == 0   # unknown prep bit
    fx = lib.kda_backward_ex
    assert fx(*ins, 1.0, None, A + (5 << 30), None, *grads, None, 1, 64, 1, 128, 128, 1, 0, 8, A + (20 << 30),
              1 << 40, None) == binding.KDA_ERR_INVALID_ARG                # unknown prep bit
    assert fx(*ins, 1.0, None, A + (5 << 30), None, *grads, None, 1, 64, 1, 128, 128, 1, 0, 7, A + (20 << 30),
              one, None) == binding.KDA_ERR_INVALID_ARG                    # no room for the prepared inputs
    assert call(wsb=one - 1) == binding.KDA_ERR_INVALID_ARG           # below one (sequence, head)'s records
    # a 256-byte error-word header, then the records of every (sequence, head)
    assert lib.kda_backward_workspace_size(2, 64, 3, 128, 128, 1) == 256 + 6 * (one - 256)
    bad = list(grads)
    bad[0] = A + 64                                                   # grad_q overlaps q
    assert call(grads=bad) == binding.KDA_ERR_INVALID_ARG
    bad = list(grads)
    bad[1] = A + (10 << 30) + 256                                     # grad_k overlaps grad_q
    assert call(grads=bad) == binding.KDA_ERR_INVALID_ARG
    bad = list(grads)
    bad[3] = None                                                     # per-channel gate needs grad_g
    assert call(grads=bad) == binding.KDA_ERR_INVALID_ARG
    assert call(grad_o=None) == binding.KDA_ERR_INVALID_ARG
    assert f(*ins, 1.0, None, A + (5 << 30), None, *grads, None, 0, 64, 1, 128, 128, 1, 0, None, 0, None) \
        == binding.KDA_OK                                             # B = 0 with nothing to copy
