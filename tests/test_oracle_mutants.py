"""Plants plausible slips in a private copy of the oracle (on the CPU) and
checks that the pins catch every one of them."""
import os
import subprocess

import pytest

import oracle
from tests import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")

# (name, text in the oracle, replacement): each is a slip someone could make.
MUTANTS = [
    ("delta_sign", "u[j] = bt * (vt[j0 + j] - pred);", "u[j] = bt * (vt[j0 + j] + pred);"),
    ("beta_dropped", "u[j] = bt * (vt[j0 + j] - pred);", "u[j] = (vt[j0 + j] - pred);"),
    ("predict_with_q", "pred += S[(size_t)i * nc + j] * kt[i];", "pred += S[(size_t)i * nc + j] * qt[i];"),
    ("write_with_q", "S[(size_t)i * nc + j] += kt[i] * u[j];", "S[(size_t)i * nc + j] += qt[i] * u[j];"),
    ("scale_dropped", "o[tok * dv + j0 + j] = scale * acc;", "o[tok * dv + j0 + j] = acc;"),
    ("gate_sign", "a[i] = exp(gt[i]);", "a[i] = exp(-gt[i]);"),
    ("gate_on_columns", "S[(size_t)i * nc + j] *= a[i];", "S[(size_t)i * nc + j] *= a[j % dk];"),
]


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    mutated = src.replace(old, new)
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(mutated)
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(so), str(c), "-lm"],
                   check=True)
    return oracle.bind(str(so))


def _pin_errors(lib):
    fwd = lambda *a, **kw: oracle.kda_forward(*a, lib=lib, **kw)
    return {p.__name__: p(fwd) for p in oracle_pins.ALL_PINS}


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    errs = _pin_errors(_build_mutant(tmp_path, name, old, new))
    assert max(errs.values()) > 1e-6, f"no pin caught mutant {name}: {errs}"


def test_output_read_before_write_is_caught(tmp_path):
    """Moving the output read ahead of the rank-1 write (o from S' instead of S_t)."""
    src = open(SRC).read()
    read_block = src[src.index("    /* o_t = scale * S_t^T q_t */"):src.index("  }\n\n  if (sT)")]
    write_block = src[src.index("    /* S = S' + k u^T */"):src.index("    /* o_t = scale * S_t^T q_t */")]
    mutated = src.replace(write_block + read_block, read_block + write_block)
    assert mutated != src
    c = tmp_path / "rbw.c"
    so = tmp_path / "librbw.so"
    c.write_text(mutated)
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(so), str(c), "-lm"],
                   check=True)
    errs = _pin_errors(oracle.bind(str(so)))
    assert max(errs.values()) > 1e-6, errs


def test_delta_before_decay_is_caught(tmp_path):
    """Taking the delta correction against the undecayed state (the gate applied
    after the prediction instead of before it)."""
    src = open(SRC).read()
    decay = src[src.index("    /* S' = Diag(exp(g_t)) S"):src.index("    /* u = beta (v - S'^T k)")]
    delta = src[src.index("    /* u = beta (v - S'^T k)"):src.index("    /* S = S' + k u^T */")]
    mutated = src.replace(decay + delta, delta + decay)
    assert mutated != src
    c = tmp_path / "dbd.c"
    so = tmp_path / "libdbd.so"
    c.write_text(mutated)
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(so), str(c), "-lm"],
                   check=True)
    errs = _pin_errors(oracle.bind(str(so)))
    assert max(errs.values()) > 1e-6, errs
