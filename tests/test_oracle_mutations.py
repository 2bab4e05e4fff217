"""The pins must catch plausible slips in the oracle.

Each case below edits a copy of ``oracle/kda_oracle.c`` on the CPU (a dropped
term, a wrong sign, index or operand, a misplaced eps, a step out of order),
compiles it to a temporary shared object, swaps it in for the real oracle and
runs every pin of ``test_oracle_pins.py``: at least one pin must fail.
"""
import inspect
import os
import re
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins


def _swap_steps_4_and_5(src: str) -> str:
    a = src.index("/* 4. S += k u^T */")
    b = src.index("/* 5. o = scale S^T q")
    c = src.index("/* 6. optional gated RMS norm")
    return src[:a] + src[b:c] + src[a:b] + src[c:]


MUTANTS = {
    "no_decay": ("S[i * V + j] *= d;", "S[i * V + j] *= 1.0;"),
    "decay_by_value_column": ("S[i * V + j] *= d;", "S[i * V + j] *= exp((double)gt[j % K]);"),
    "no_beta": ("u[j] = bt * (", "u[j] = 1.0 * ("),
    "sign_of_correction": ("(bf16_to_double(vt[j]) - rk[j])", "(rk[j] - bf16_to_double(vt[j]))"),
    "correction_reads_q": ("acc += S[i * V + j] * bf16_to_double(kt[i]);",
                           "acc += S[i * V + j] * bf16_to_double(qt[i]);"),
    "transposed_state": ("acc += S[i * V + j] * bf16_to_double(kt[i]);",
                         "acc += S[j * K + i] * bf16_to_double(kt[i]);"),
    "update_writes_q": ("const double ki = bf16_to_double(kt[i]);",
                        "const double ki = bf16_to_double(qt[i]);"),
    "no_scale": ("ot[j] = scale * acc;", "ot[j] = acc;"),
    "readout_before_update": _swap_steps_4_and_5,
    "token_stride_q": ("const uint16_t *qt = q + t * q_tstride;", "const uint16_t *qt = q;"),
    "token_stride_g": ("const double *gt = g + t * g_tstride;", "const double *gt = g;"),
    "head_stride_beta": ("beta + (n * T * HV + h)", "beta + (n * T * HV)"),
    "slot_ignores_head": ("(((int64_t)slot * HV + h) * K * V)", "(((int64_t)slot * HV) * K * V)"),
    "gate_sign": ("exp(-bf16_to_double(zt[j]))", "exp(bf16_to_double(zt[j]))"),
    "eps_outside_sqrt": ("1.0 / sqrt(ss / (double)V + eps)", "1.0 / (sqrt(ss / (double)V) + eps)"),
    "sum_not_mean": ("ss / (double)V + eps", "ss + eps"),
    "no_norm_weight": (" * bf16_to_double(w[j]) * gate", " * gate"),
    "bf16_truncates": ("const double q = nearbyint(ldexp(a, -lsb));", "const double q = floor(ldexp(a, -lsb));"),
    "bf16_ties_away": ("const double q = nearbyint(ldexp(a, -lsb));", "const double q = round(ldexp(a, -lsb));"),
    "bf16_no_subnormal": ("if (lsb < -133) lsb = -133;", "if (lsb < -200) lsb = -200;"),
    "gate_no_dt_bias": ("+ (double)dt_bias[h * K + i]", "+ 0.0 * dt_bias[h * K + i]"),
    "gate_sign_flip": ("g[e] = -a * softplus(", "g[e] = a * softplus("),
    "gate_exp_not_softplus": ("static double softplus(double x) { return x > 0.0 ? x + log1p(exp(-x)) : log1p(exp(x)); }",
                              "static double softplus(double x) { return exp(x); }"),
    "gate_a_not_exp": ("const double a = exp((double)A_log[h]);", "const double a = (double)A_log[h];"),
    "beta_sign": ("beta[r * HV + h] = 1.0 / (1.0 + exp(-bf16_to_double(", "beta[r * HV + h] = 1.0 / (1.0 + exp(bf16_to_double("),
}


def _pin_functions():
    return [f for name, f in inspect.getmembers(pins, inspect.isfunction)
            if name.startswith("test_") and not inspect.signature(f).parameters
            or name == "test_gated_rank1_closed_form"]


def _run_pins() -> list[str]:
    failed = []
    for f in _pin_functions():
        kwargs = {"eps": 1e-6} if "eps" in inspect.signature(f).parameters else {}
        try:
            f(**kwargs)
        except (AssertionError, ValueError):
            failed.append(f.__name__)
    return failed


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path, monkeypatch):
    src = open(oracle._SRC).read()
    m = MUTANTS[name]
    if callable(m):
        mutated = m(src)
    else:
        assert src.count(m[0]) >= 1, f"mutation anchor missing: {m[0]}"
        mutated = src.replace(m[0], m[1])
    assert mutated != src
    c_path = tmp_path / "mutant.c"
    c_path.write_text(mutated)
    so_path = str(tmp_path / "libmutant.so")
    subprocess.check_call(["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fPIC", "-shared",
                           "-o", so_path, str(c_path), "-lm"])
    monkeypatch.setattr(oracle, "_lib", oracle.load_library(so_path))
    failed = _run_pins()
    assert failed, f"no pin caught mutant {name}"


def test_unmutated_oracle_passes_every_pin():
    assert _run_pins() == []
