"""The pins must catch plausible mistakes in the oracle.

Each case compiles a copy of ``oracle/kda_oracle.c`` with one deliberate
mistake (a dropped term, a wrong sign, a wrong operand or index) into a
temporary directory, runs the independent checks against it, and requires at
least one of them to fail.  The real oracle passes the same checks.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle
from _closed_form import chunked, product_form_unit
from kda_delta_rule_chunkwise_b200 import inputs as kin

SRC = os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")

MUTANTS = {
    "no_decay": ("const double a = exp(gc);", "const double a = 1.0;"),
    "wrong_sign_delta": ("A_kT[j] = bt * (vt[j] - A_kT[j]);",
                         "A_kT[j] = bt * (vt[j] + A_kT[j]);"),
    "dropped_beta": ("A_kT[j] = bt * (vt[j] - A_kT[j]);",
                     "A_kT[j] = (vt[j] - A_kT[j]);"),
    "no_clamp": ("const double gc = gt[c] < -5.0 ? -5.0 : gt[c];",
                 "const double gc = gt[c];"),
    "predict_with_q": ("for (int j = 0; j < dv; ++j) A_kT[j] += row[j] * kc;",
                       "for (int j = 0; j < dv; ++j) A_kT[j] += row[j] * qt[c];"),
    "readout_with_k": ("ot[j] += row[j] * qc;", "ot[j] += row[j] * kt[c];"),
    "stale_query_index": ("const double *qt = J->q + ((size_t)t * H + h) * dk;",
                          "const double *qt = J->q + ((size_t)(t > t0 ? t - 1 : t) * H + h) * dk;"),
    "ignores_state_in": ("if (J->state_in)\n", "if (0)\n"),
    "transposed_write": ("row[j] += kc * A_kT[j];", "row[j] += A_kT[c % dv] * kt[j % dk];"),
    "decay_twice": ("for (int j = 0; j < dv; ++j) row[j] *= a;",
                    "for (int j = 0; j < dv; ++j) row[j] *= a * a;"),
}


def _build(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    path_c = tmp_path / f"{name}.c"
    path_c.write_text(src.replace(old, new))
    so = tmp_path / f"lib{name}.so"
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread",
                    "-o", str(so), str(path_c), "-lm"], check=True)
    return oracle.load_library(str(so))


def _checks(lib):
    """Independent checks; returns the list of names that failed."""
    failed = []
    inp = kin.prefill_inputs(1, 70, 2, 6, 6, "f32", seed=21, state="normal")
    f = lambda x: x.double().numpy()
    q, k, v, g, b, s0 = (f(x) for x in (inp.q, inp.k, inp.v, inp.g, inp.beta, inp.state_in))
    g = g.copy()
    g[0, ::5, :, 0] = -7.5          # below the bound: must act as -5
    o, s = oracle.recurrence(q, k, v, g, b, s0, lib=lib)
    rs = lambda x: x.reshape((-1,) + x.shape[2:])
    oc, sc = chunked(rs(q), rs(k), rs(v), rs(g), rs(b), s0, np.array([0, 70]), 16)
    if not np.allclose(o.reshape(oc.shape), oc, atol=1e-10, rtol=0):
        failed.append("chunked_o")
    if not np.allclose(s, sc, atol=1e-10, rtol=0):
        failed.append("chunked_state")
    O, S = product_form_unit(q[0, :, 1], k[0, :, 1], v[0, :, 1], g[0, :, 1], b[0, :, 1],
                             s0[0, 1])
    if not np.allclose(o[0, :, 1], O, atol=1e-10, rtol=0):
        failed.append("product_form")
    return failed


def test_real_oracle_passes_mutation_checks():
    assert _checks(None) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    lib = _build(tmp_path, name, old, new)
    assert _checks(lib), f"mutant {name} was not detected by any pin"
