"""fp64 CPU oracle for Kimi Delta Attention (KDA) -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It is the plain token-by-token
recurrence (KimiLinear article, section 2.3, KDA state-update rule) written in
C (``kda_oracle.c``) and shares nothing with the CUDA library.

Pins (tests/test_oracle_pins.py) tie it to facts other than itself: the
gated/plain linear-attention closed form, dense brute-force products of the
transition matrices on T <= 8, exact retrieval under the delta rule, the
DeltaNet and Gated DeltaNet special cases, boundedness, and hand-derived
worked examples under tests/golden/.  ``prepare_inputs`` (fused input
preparation: unit-length q and k, log-sigmoid gates, sigmoid write
strengths) is pinned in tests/test_oracle_prep.py against closed forms and
a second formula for each step.  ``kda_backward`` (reverse-mode gradients of
the recurrence) is pinned in tests/test_oracle_backward.py by central
differences of ``kda_forward`` and by torch autograd through a plain fp64
loop; ``prepare_backward`` (the chain rule through the preparation) in
tests/test_oracle_prep_backward.py by central differences of
``prepare_inputs`` and of the prepared forward.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")

MODE_DELTA = 0   # the KDA recurrence
MODE_LINEAR = 1  # delta correction dropped: gated linear attention (pinning aid)

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE fp64, no fast-math) and return the .so path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"],
                       check=True)
        os.replace(tmp, _LIB)
    return _LIB


def bind(path: str):
    """Load an oracle shared object from ``path`` and declare its signatures."""
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.kda_oracle_forward.argtypes = [dp, dp, dp, dp, dp, ctypes.c_double, dp, dp, dp] + [ctypes.c_int] * 7
    lib.kda_oracle_forward.restype = ctypes.c_int
    lib.kda_oracle_max_threads.argtypes = []
    lib.kda_oracle_max_threads.restype = ctypes.c_int
    lib.kda_oracle_backward.argtypes = [dp] * 5 + [ctypes.c_double] + [dp] * 9 + [ctypes.c_int] * 6
    lib.kda_oracle_backward.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = bind(build())
    return _lib


def _as_f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor (any dtype, any device): exact upcast to fp64
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def max_threads() -> int:
    return int(_load().kda_oracle_max_threads())


def kda_forward(q, k, v, g, beta, scale, initial_state=None, mode=MODE_DELTA, nthreads=0,
                want_state=True, lib=None):
    """Token-by-token fp64 KDA over [B,T,H,d] inputs.

    Returns (o [B,T,H,dv] fp64, final_state [B,H,dk,dv] fp64 or None).
    Inputs may be numpy arrays or torch tensors of any float dtype; they are
    upcast exactly to fp64, so the oracle sees the values the GPU reads.
    """
    q, k, v, g, beta = (_as_f64(x) for x in (q, k, v, g, beta))
    s0 = _as_f64(initial_state)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == (B, T, H, dk) and g.shape == (B, T, H, dk)
    assert v.shape == (B, T, H, dv) and beta.shape == (B, T, H)
    if s0 is not None:
        assert s0.shape == (B, H, dk, dv)
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    sT = np.zeros((B, H, dk, dv), dtype=np.float64) if want_state else None
    rc = (lib or _load()).kda_oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                                    _ptr(s0), _ptr(o), _ptr(sT), B, T, H, dk, dv, int(mode),
                                    int(nthreads))
    if rc != 0:
        raise ValueError("kda_oracle_forward rejected its arguments")
    return o, sT


def kda_decode(q, k, v, g, beta, scale, state, nthreads=0):
    """Decode steps: inputs [S,N,H,d] for S consecutive single-token steps.

    The decode step is the same recurrence with one token per call, so it is
    the forward pass with T = S on a [N,S,H,d] view (each sequence carries its
    own state).  Returns (o [S,N,H,dv], final state [N,H,dk,dv]).
    """
    q, k, v, g, beta = (_as_f64(x) for x in (q, k, v, g, beta))
    tr = lambda x: np.ascontiguousarray(np.swapaxes(x, 0, 1))
    o, sT = kda_forward(tr(q), tr(k), tr(v), tr(g), tr(beta), scale, state, nthreads=nthreads)
    return np.ascontiguousarray(np.swapaxes(o, 0, 1)), sT


# Fused input preparation (kda_prep bits of the C ABI).  The pages give no
# formula for these steps; they are the transforms that make raw projections
# into the operator's inputs (unit-length q and k, log-gates <= 0, write
# strengths in (0, 1)), written out in fp64 from their definitions.
PREP_L2NORM_QK, PREP_GATE_LOGSIGMOID, PREP_BETA_SIGMOID = 1, 2, 4
L2_EPS = 1e-6


def prepare_inputs(q, k, g, beta, prep):
    """(q, k, g, beta) in fp64 after the preparation steps selected by ``prep``:
    q <- q / sqrt(sum_c q_c^2 + 1e-6) (same for k) per token and head,
    g <- log sigmoid(g) = min(g, 0) - log(1 + exp(-|g|)), beta <- 1 / (1 + exp(-beta)).
    g may be None (no gate)."""
    q, k, beta = _as_f64(q), _as_f64(k), _as_f64(beta)
    g = None if g is None else _as_f64(g)
    if prep & PREP_L2NORM_QK:
        q = q / np.sqrt(np.sum(q * q, axis=-1, keepdims=True) + L2_EPS)
        k = k / np.sqrt(np.sum(k * k, axis=-1, keepdims=True) + L2_EPS)
    if prep & PREP_GATE_LOGSIGMOID and g is not None:
        g = np.minimum(g, 0.0) - np.log1p(np.exp(-np.abs(g)))
    if prep & PREP_BETA_SIGMOID:
        beta = 1.0 / (1.0 + np.exp(-beta))
    return q, k, g, beta


def prepare_backward(q, k, g, beta, prep, dq_hat, dk_hat, dg_hat, dbeta_hat):
    """Gradients with respect to the raw inputs of prepare_inputs, given the
    gradients (dq_hat, dk_hat, dg_hat, dbeta_hat) with respect to its
    outputs (the chain rule of each preparation step, fp64):
    q_hat = r q with r = (sum_c q_c^2 + 1e-6)^-1/2:  dq = r (dq_hat - q_hat (q_hat . dq_hat));
    g_hat = log sigmoid(g):  dg = dg_hat sigmoid(-g);
    beta_hat = sigmoid(beta):  dbeta = dbeta_hat sigmoid(beta) (1 - sigmoid(beta)).
    Steps whose bit is not set pass their gradient through; g may be None."""
    q, k, beta = _as_f64(q), _as_f64(k), _as_f64(beta)
    dq, dk, dbeta = _as_f64(dq_hat), _as_f64(dk_hat), _as_f64(dbeta_hat)
    dg = None if dg_hat is None else _as_f64(dg_hat)
    if prep & PREP_L2NORM_QK:
        out = []
        for x, dx in ((q, dq), (k, dk)):
            r = 1.0 / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + L2_EPS)
            xh = x * r
            out.append(r * (dx - xh * np.sum(xh * dx, axis=-1, keepdims=True)))
        dq, dk = out
    if prep & PREP_GATE_LOGSIGMOID and dg is not None:
        dg = dg / (1.0 + np.exp(_as_f64(g)))            # sigmoid(-g)
    if prep & PREP_BETA_SIGMOID:
        sb = 1.0 / (1.0 + np.exp(-beta))
        dbeta = dbeta * sb * (1.0 - sb)
    return dq, dk, dg, dbeta


def kda_backward(q, k, v, g, beta, scale, initial_state, d_o, d_final_state=None, nthreads=0, lib=None):
    """fp64 gradients of a loss through kda_forward, given dL/do [B,T,H,dv] and
    dL/dS_T [B,H,dk,dv] (None: zero).  Returns a dict with dq, dk, dv, dg
    (per key channel), dbeta and dS0 (fp64 numpy arrays, the inputs' layouts).
    Reverse-mode differentiation of the token-by-token recurrence, column by
    column of the state (kda_oracle.c, kda_oracle_backward)."""
    lib = lib or _load()
    q, k, v, g, beta, d_o = (_as_f64(x) for x in (q, k, v, g, beta, d_o))
    s0, dsT = _as_f64(initial_state), _as_f64(d_final_state)
    B, T, H, nk = q.shape
    nv = v.shape[-1]
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v), dg=np.zeros_like(g),
               dbeta=np.zeros_like(beta), dS0=np.zeros((B, H, nk, nv)))
    rc = lib.kda_oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(s0),
                                 _ptr(d_o), _ptr(dsT), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                                 _ptr(out["dg"]), _ptr(out["dbeta"]), _ptr(out["dS0"]), B, T, H, nk, nv,
                                 int(nthreads))
    if rc != 0:
        raise ValueError("kda_oracle_backward rejected its arguments")
    return out
