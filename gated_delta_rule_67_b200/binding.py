"""Thin Python binding of libkda.so (include/kda.h): argument marshalling only.

Every step of the operator runs in the library's CUDA kernels; this module
checks tensor placement/dtype/contiguity, allocates outputs and workspace
with torch when the caller did not pass them, and forwards raw device
pointers plus the current CUDA stream.  There is no CPU fallback: without
the compiled library or a CUDA device every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkda.so")

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_CUDA, KDA_ERR_TIMEOUT = range(5)
KDA_F32, KDA_BF16 = 0, 1

# Every symbol include/kda.h declares, with (restype, argtypes).
_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "kda_status_string": (ctypes.c_char_p, [_i]),
    "kda_version": (_i, []),
    "kda_chunk_fwd_workspace_size": (_sz, [_i] * 7),
    "kda_chunk_fwd_launch_count": (_i, [_i] * 7),
    "kda_chunk_fwd": (_i, [_vp] * 5 + [_f, _vp, _vp, _vp] + [_i] * 7 + [_vp, _sz, _vp]),
    "kda_chunk_fwd_profiled": (_i, [_vp] * 5 + [_f, _vp, _vp, _vp] + [_i] * 7 + [_vp, _sz, _vp, _vp]),
    "kda_chunk_fwd_noalloc": (_i, [_vp] * 5 + [_f, _vp, _vp, _vp] + [_i] * 7 + [_vp]),
    "kda_chunk_fwd_check": (_i, [_vp, _sz, _vp]),
    "kda_chunk_fwd_noalloc_check": (_i, [_vp]),
    "kda_wait_selftest": (_i, [_vp, _sz, _vp]),
    "kda_recurrent_step": (_i, [_vp] * 5 + [_f, _vp, _vp] + [_i] * 5 + [_vp]),
    "kda_chunk_fwd_ex": (_i, [_vp] * 5 + [_f, _vp, _vp, _vp] + [_i] * 9 + [_vp, _sz, _vp]),
    "kda_recurrent_step_ex": (_i, [_vp] * 5 + [_f, _vp, _vp] + [_i] * 7 + [_vp]),
    "kda_backward_workspace_size": (_sz, [_i] * 6),
    "kda_backward": (_i, [_vp] * 5 + [_f] + [_vp] * 9 + [_i] * 7 + [_vp, _sz, _vp]),
    "kda_backward_ex_workspace_size": (_sz, [_i] * 7),
    "kda_backward_ex": (_i, [_vp] * 5 + [_f] + [_vp] * 9 + [_i] * 8 + [_vp, _sz, _vp]),
}

# kda_gate: how the forget gate enters the update (see include/kda.h)
KDA_GATE_CHANNEL, KDA_GATE_HEAD, KDA_GATE_NONE = 0, 1, 2
# kda_prep bits: raw inputs prepared inside the kernels (see include/kda.h)
KDA_PREP_L2NORM_QK, KDA_PREP_GATE_LOGSIGMOID, KDA_PREP_BETA_SIGMOID = 1, 2, 4
KDA_PREP_ALL = KDA_PREP_L2NORM_QK | KDA_PREP_GATE_LOGSIGMOID | KDA_PREP_BETA_SIGMOID


def _gate_kind(g, lead):
    """Gate kind from g's shape: per key channel [*lead, dk] (KDA), per head
    [*lead] (Gated DeltaNet), or None (DeltaNet)."""
    if g is None:
        return KDA_GATE_NONE
    if tuple(g.shape) == tuple(lead):
        return KDA_GATE_HEAD
    return KDA_GATE_CHANNEL

_lib = None


class KDAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def load(path: str = LIB_PATH):
    """Load libkda.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"libkda.so not built at {path}; run gated_delta_rule_67_b200.build.build()")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype, fn.argtypes = res, args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().kda_status_string(int(status)).decode()


def version() -> int:
    return int(load().kda_version())


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return KDA_F32
    if t == torch.bfloat16:
        return KDA_BF16
    raise TypeError(f"unsupported dtype {t}; KDA takes float32 or bfloat16")


def _check_dev(name, x, dtype=None):
    if not isinstance(x, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not x.is_cuda:
        raise ValueError(f"{name} must live on a CUDA device (no CPU path exists)")
    if not x.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and x.dtype != dtype:
        raise TypeError(f"{name} has dtype {x.dtype}, expected {dtype}")


def _ptr(x):
    return None if x is None else ctypes.c_void_p(x.data_ptr())


def _stream(stream, device):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _on(device):
    """Makes the tensors' device current for the C call: the library keys its
    per-device set-up (function attributes, the static scratch) by the
    current device, which must own the buffers and the stream."""
    return torch.cuda.device(device)


def kda_chunk_fwd_workspace_size(B, T, H, dk, dv, chunk=64, dtype=torch.bfloat16) -> int:
    return int(load().kda_chunk_fwd_workspace_size(B, T, H, dk, dv, chunk, _dtype_code(dtype)))


def kda_chunk_fwd_launch_count(B, T, H, dk, dv, chunk=64, dtype=torch.bfloat16) -> int:
    """Kernels one kda_chunk_fwd call with these arguments launches (-1: rejected)."""
    return int(load().kda_chunk_fwd_launch_count(B, T, H, dk, dv, chunk, _dtype_code(dtype)))


def kda_chunk_fwd(q, k, v, g, beta, scale=None, initial_state=None, *, chunk=64, o=None, final_state=None,
                  output_final_state=True, workspace=None, stream=None, events=None, prep=0):
    """Chunked KDA prefill.  q,k [B,T,H,dk], v [B,T,H,dv], beta [B,T,H] (fp32 or bf16, CUDA).

    g selects the forget gate: [B,T,H,dk] per key channel (KDA), [B,T,H] one
    per head (Gated DeltaNet), or None (DeltaNet, no forgetting).
    ``prep``: KDA_PREP_* bits; the marked inputs are raw projections prepared
    in the kernels (q, k to unit length; g = logsigmoid(g); beta = sigmoid(beta)).
    Returns (o [B,T,H,dv] in the input dtype, final_state [B,H,dk,dv] fp32 or None).
    ``final_state`` may be ``initial_state`` itself for an in-place update.
    ``events``: optional three recorded torch.cuda.Event objects; the library
    records them before, between and after its kernels (kda_chunk_fwd_profiled,
    per-channel gates only).
    """
    lib = load()
    for name, x in (("q", q), ("k", k), ("v", v), ("beta", beta)):
        _check_dev(name, x, q.dtype)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    gate = _gate_kind(g, (B, T, H))
    if g is not None:
        _check_dev("g", g, q.dtype)
    if k.shape != q.shape or (gate == KDA_GATE_CHANNEL and g.shape != q.shape) or v.shape[:3] != (B, T, H) \
            or beta.shape != (B, T, H):
        raise ValueError("shape mismatch among q, k, v, g, beta")
    if scale is None:
        scale = dk ** -0.5
    code = _dtype_code(q.dtype)
    if initial_state is not None:
        _check_dev("initial_state", initial_state, torch.float32)
        if initial_state.shape != (B, H, dk, dv):
            raise ValueError("initial_state must be [B,H,dk,dv]")
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    _check_dev("o", o, q.dtype)
    if final_state is None and output_final_state:
        final_state = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    if final_state is not None:
        _check_dev("final_state", final_state, torch.float32)
    need = int(lib.kda_chunk_fwd_workspace_size(B, T, H, dk, dv, chunk, code))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(initial_state), _ptr(o),
            _ptr(final_state), B, T, H, dk, dv, chunk, code, _ptr(workspace), ws_bytes, _stream(stream, q.device))
    if gate != KDA_GATE_CHANNEL or prep:
        if events is not None:
            raise ValueError("events are recorded for prepared per-channel-gate inputs only")
        with _on(q.device):
            st = lib.kda_chunk_fwd_ex(*args[:16], gate, int(prep), *args[16:])
    elif events is None:
        with _on(q.device):
            st = lib.kda_chunk_fwd(*args)
    else:
        if len(events) != 3:
            raise ValueError("events must hold three torch.cuda.Event objects")
        handles = (ctypes.c_void_p * 3)(*[ev.cuda_event for ev in events])
        with _on(q.device):
            st = lib.kda_chunk_fwd_profiled(*args, handles)
    if st != KDA_OK:
        raise KDAError(st, "kda_chunk_fwd")
    return o, final_state


def kda_chunk_fwd_noalloc(q, k, v, g, beta, scale=None, initial_state=None, *, chunk=64, o=None,
                          final_state=None, output_final_state=True, stream=None):
    """kda_chunk_fwd using the library's static device scratch instead of a
    workspace: for callers that cannot allocate device memory.  Fits problems
    whose workspace is at most 64 MiB (about 900 chunk-heads, bf16); calls
    overlapping on the GPU race."""
    lib = load()
    for name, x in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta)):
        _check_dev(name, x, q.dtype)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or g.shape != q.shape or v.shape[:3] != (B, T, H) or beta.shape != (B, T, H):
        raise ValueError("shape mismatch among q, k, v, g, beta")
    if scale is None:
        scale = dk ** -0.5
    if initial_state is not None:
        _check_dev("initial_state", initial_state, torch.float32)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    _check_dev("o", o, q.dtype)
    if final_state is None and output_final_state:
        final_state = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    with _on(q.device):
        st = lib.kda_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                                       _ptr(initial_state), _ptr(o), _ptr(final_state), B, T, H, dk, dv, chunk,
                                       _dtype_code(q.dtype), _stream(stream, q.device))
    if st != KDA_OK:
        raise KDAError(st, "kda_chunk_fwd_noalloc")
    return o, final_state


def kda_chunk_fwd_check(workspace, stream=None) -> int:
    """Status word a bounded on-device wait may have left in ``workspace`` (synchronises)."""
    if workspace is None:
        return KDA_OK
    with _on(workspace.device):
        return int(load().kda_chunk_fwd_check(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                              _stream(stream, workspace.device)))


def kda_chunk_fwd_noalloc_check(device=None, stream=None) -> int:
    """Status word of the static scratch after kda_chunk_fwd_noalloc calls on
    ``device`` (default: the current device); synchronises.  KDA_OK, or
    KDA_ERR_TIMEOUT if a bounded on-device wait of the last call gave up."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with _on(device):
        return int(load().kda_chunk_fwd_noalloc_check(_stream(stream, device)))


def kda_wait_selftest(workspace, stream=None) -> int:
    """Runs the bounded-wait failure path on the device (see include/kda.h); returns the status
    kda_chunk_fwd_check reads afterwards (KDA_ERR_TIMEOUT when the mechanism works)."""
    lib = load()
    nbytes = workspace.numel() * workspace.element_size()
    with _on(workspace.device):
        st = lib.kda_wait_selftest(_ptr(workspace), nbytes, _stream(stream, workspace.device))
    if st != KDA_OK:
        raise KDAError(st, "kda_wait_selftest")
    return kda_chunk_fwd_check(workspace, stream)


def kda_recurrent_step(q, k, v, g, beta, state, scale=None, *, o=None, stream=None, prep=0):
    """One decode step.  q,k [N,H,dk], v [N,H,dv], beta [N,H]; state [N,H,dk,dv] fp32 updated in place.

    g selects the forget gate: [N,H,dk] per key channel (KDA), [N,H] one per
    head (Gated DeltaNet), or None (DeltaNet).  ``prep``: KDA_PREP_* bits as for
    kda_chunk_fwd.  Returns o [N,H,dv] in the input dtype.
    """
    lib = load()
    for name, x in (("q", q), ("k", k), ("v", v), ("beta", beta)):
        _check_dev(name, x, q.dtype)
    _check_dev("state", state, torch.float32)
    N, H, dk = q.shape
    dv = v.shape[-1]
    gate = _gate_kind(g, (N, H))
    if g is not None:
        _check_dev("g", g, q.dtype)
    if k.shape != q.shape or (gate == KDA_GATE_CHANNEL and g.shape != q.shape) or v.shape[:2] != (N, H) \
            or beta.shape != (N, H):
        raise ValueError("shape mismatch among q, k, v, g, beta")
    if state.shape != (N, H, dk, dv):
        raise ValueError("state must be [N,H,dk,dv]")
    if scale is None:
        scale = dk ** -0.5
    if o is None:
        o = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    _check_dev("o", o, q.dtype)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(state), _ptr(o), N, H, dk, dv,
            _dtype_code(q.dtype))
    with _on(q.device):
        if gate == KDA_GATE_CHANNEL and not prep:
            st = lib.kda_recurrent_step(*args, _stream(stream, q.device))
        else:
            st = lib.kda_recurrent_step_ex(*args, gate, int(prep), _stream(stream, q.device))
    if st != KDA_OK:
        raise KDAError(st, "kda_recurrent_step")
    return o


def kda_backward(q, k, v, g, beta, grad_o, scale=None, initial_state=None, grad_final_state=None, *,
                 workspace=None, stream=None, want_initial_state_grad=True, prep=0):
    """Gradients of a loss through kda_chunk_fwd (g per key channel [B,T,H,dk],
    per head [B,T,H] or None, as for the forward), given grad_o = dL/do
    [B,T,H,dv] and grad_final_state = dL/dS_T [B,H,dk,dv] fp32 (or None).
    ``prep``: the forward's KDA_PREP_* bits; q, k, g, beta are then the raw
    inputs and the gradients are taken with respect to them.

    Returns a dict: dq, dk, dv, dg (like g; None without a gate), dbeta (input
    dtype) and dS0 = dL/dS_0 fp32 (None if not wanted).
    """
    lib = load()
    for name, x in (("q", q), ("k", k), ("v", v), ("beta", beta), ("grad_o", grad_o)):
        _check_dev(name, x, q.dtype)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    gate = _gate_kind(g, (B, T, H))
    if g is not None:
        _check_dev("g", g, q.dtype)
    if k.shape != q.shape or (gate == KDA_GATE_CHANNEL and g.shape != q.shape) or v.shape[:3] != (B, T, H) \
            or beta.shape != (B, T, H) or grad_o.shape != v.shape:
        raise ValueError("shape mismatch among q, k, v, g, beta, grad_o")
    if scale is None:
        scale = dk ** -0.5
    for name, x in (("initial_state", initial_state), ("grad_final_state", grad_final_state)):
        if x is not None:
            _check_dev(name, x, torch.float32)
            if x.shape != (B, H, dk, dv):
                raise ValueError(f"{name} must be [B,H,dk,dv]")
    code = _dtype_code(q.dtype)
    out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
               dg=None if g is None else torch.empty_like(g), dbeta=torch.empty_like(beta),
               dS0=torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device) if want_initial_state_grad
               else None)
    need = int(lib.kda_backward_ex_workspace_size(B, T, H, dk, dv, code, int(prep)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with _on(q.device):
        st = lib.kda_backward_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(initial_state),
                                 _ptr(grad_o), _ptr(grad_final_state), _ptr(out["dq"]), _ptr(out["dk"]),
                                 _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dbeta"]), _ptr(out["dS0"]), B, T, H, dk,
                                 dv, code, gate, int(prep), _ptr(workspace), ws_bytes, _stream(stream, q.device))
    if st != KDA_OK:
        raise KDAError(st, "kda_backward")
    return out
