"""Pin sensitivity: plausible mistakes planted in a copy of the oracle fail a pin.

Each mutant is a textual edit of ``oracle/mlstm_oracle.c`` (a dropped term, a
wrong sign, a stale index, a missing scale), compiled with gcc into a
temporary directory.  The real oracle is untouched; nothing runs on a GPU.
"""
import functools
import os
import subprocess

import pytest

import oracle
import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "mlstm_oracle.c")

MUTANTS = {
    "stabiliser_drops_forget": ("fmax(lf + m, li)", "fmax(m, li)"),
    "forget_factor_sign": ("exp(lf + m - m_new)", "exp(lf - m - m_new)"),
    "input_factor_stale_m": ("exp(li - m_new)", "exp(li - m)"),
    "missing_key_scale": ("ks[a] = s * k[a];", "ks[a] = k[a];"),
    "lower_bound_sign": ("exp(-m_new)", "exp(m_new)"),
    "denominator_not_abs": ("fmax(fabs(den),", "fmax((den),"),
    "denominator_uses_key": ("den += n[a] * q[a];", "den += n[a] * ks[a];"),
    "logsigmoid_sign": ("if (x >= 0.0) return -log1p(exp(-x));", "if (x >= 0.0) return -log1p(exp(x));"),
    "sigmoid_mode_raw_gate": (": oracle_logsigmoid(i_pre[bh * T + t]);", ": i_pre[bh * T + t];"),
    "normaliser_no_input_gate": ("n[a] = fa * n[a] + ia * ks[a];", "n[a] = fa * n[a] + ks[a];"),
    "memory_no_forget": ("Ca[j] = fa * Ca[j] + ia * ks[a] * v[j];", "Ca[j] = Ca[j] + ia * ks[a] * v[j];"),
    "initial_stabiliser_ignored": ("m = m0[bh];", "m = 0.0;"),
}


@functools.lru_cache(maxsize=None)
def _build(name, tmpdir):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    path_c = os.path.join(tmpdir, f"{name}.c")
    path_so = os.path.join(tmpdir, f"lib{name}.so")
    with open(path_c, "w") as fh:
        fh.write(src.replace(old, new))
    subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c99", path_c, "-o",
                    path_so, "-lm"], check=True)
    return oracle.open_library(path_so)


@pytest.fixture(scope="module")
def tmpdir_str(tmp_path_factory):
    return str(tmp_path_factory.mktemp("oracle_mutants"))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_fails_a_pin(name, tmpdir_str):
    lib = _build(name, tmpdir_str)
    run = functools.partial(oracle.mlstm_recurrent, lib=lib)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(run)
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passes every pin"


# Mutants of the sigmoid-input-gate variant's oracle function (plain
# definition, no stabiliser, no normaliser); caught by pins.SIG_PLAIN_PINS.
SIG_MUTANTS = {
    "plain_input_gate_raw": ("const double ig = oracle_sigmoid(i_pre[bh * T + t]);",
                             "const double ig = i_pre[bh * T + t];"),
    "plain_no_forget": ("C[a * DV + j] = f * C[a * DV + j] + wk * v[j];",
                        "C[a * DV + j] = C[a * DV + j] + wk * v[j];"),
    "plain_missing_key_scale": ("const double wk = ig * s * k[a];",
                                "const double wk = ig * k[a];"),
    "plain_initial_frame_ignored": ("const double sc = exp(m0[bh]);", "const double sc = 1.0;"),
    "plain_sigmoid_sign": ("if (x >= 0.0) return 1.0 / (1.0 + exp(-x));",
                           "if (x >= 0.0) return 1.0 / (1.0 + exp(x));"),
}


@pytest.mark.parametrize("name", sorted(SIG_MUTANTS))
def test_sigmoid_plain_mutant_fails_a_pin(name, tmpdir_str):
    old, new = SIG_MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    path_c = os.path.join(tmpdir_str, f"{name}.c")
    path_so = os.path.join(tmpdir_str, f"lib{name}.so")
    with open(path_c, "w") as fh:
        fh.write(src.replace(old, new))
    subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c99", path_c, "-o",
                    path_so, "-lm"], check=True)
    lib = oracle.open_library(path_so)
    run = functools.partial(oracle.mlstm_sigmoid_plain, lib=lib)
    caught = []
    for pin in pins.SIG_PLAIN_PINS:
        try:
            pin(run)
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passes every pin"
