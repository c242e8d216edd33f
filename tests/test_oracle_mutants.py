"""Planted mistakes in copies of the oracle must each fail at least one pin (CPU only).

Every mutant below is a plausible slip (a dropped term, a wrong sign, a wrong index or
operand, the read-out on the wrong side of the write).  The test copies efla_oracle.c,
applies one exact text substitution, builds it into a temporary library and runs the pin
suite of oracle_pins.py on it.  The committed oracle itself is never modified.
"""
import os

import pytest

import oracle
import oracle_pins

MUTANTS = {
    "beta_instead_of_alpha": (
        "const double a = (mode == EFLA_ORACLE_EULER) ? beta[t] : efla_oracle_alpha(beta[t], lam);",
        "const double a = beta[t];"),
    "half_interval": (
        "const double a = (mode == EFLA_ORACLE_EULER) ? beta[t] : efla_oracle_alpha(beta[t], lam);",
        "const double a = (mode == EFLA_ORACLE_EULER) ? beta[t] : efla_oracle_alpha(0.5 * beta[t], lam);"),
    "gate_sign": ("return -expm1(-beta * lambda) / lambda;", "return expm1(beta * lambda) / lambda;"),
    "gate_no_denominator": ("return -expm1(-beta * lambda) / lambda;", "return -expm1(-beta * lambda);"),
    "zero_limit": ("if (lambda == 0.0)\n        return beta;", "if (lambda == 0.0)\n        return 0.0;"),
    "lambda_not_squared": ("lam += kt[i] * kt[i];", "lam += fabs(kt[i]);"),
    "write_sign": ("S[i * dv + j] -= a * kt[i] * r[j];", "S[i * dv + j] += a * kt[i] * r[j];"),
    "dropped_value": ("r[j] = -vt[j];", "r[j] = 0.0;"),
    "read_with_query": ("r[j] += kt[i] * S[i * dv + j];", "r[j] += qt[i] * S[i * dv + j];"),
    "output_before_write": ("ot[j] += qt[i] * S[i * dv + j];",
                            "ot[j] += qt[i] * (S[i * dv + j] + a * kt[i] * r[j]);"),
    "initial_state_ignored": ("if (S0)\n            memcpy(", "if (0)\n            memcpy("),
    "stale_query_index": ("const double *qt = q + t * dk;",
                          "const double *qt = q + (t > 0 ? t - 1 : 0) * dk;"),
    "stale_value_index": ("const double *vt = v + t * dv;",
                          "const double *vt = v + (t > 0 ? t - 1 : 0) * dv;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    with open(oracle.SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation target for {name} not found exactly once"
    mut_src = tmp_path / "mutant.c"
    mut_src.write_text(src.replace(old, new))
    lib = oracle.load(oracle.build(str(mut_src), str(tmp_path / "mutant.so"), force=True))
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {name!r}"


def test_unmutated_copy_passes(tmp_path):
    """Control: the same build route on an unmodified copy passes every pin."""
    with open(oracle.SRC) as f:
        src = f.read()
    p = tmp_path / "copy.c"
    p.write_text(src)
    lib = oracle.load(oracle.build(str(p), str(tmp_path / "copy.so"), force=True))
    for pin in oracle_pins.ALL_PINS:
        pin(lib)
    assert os.path.exists(tmp_path / "copy.so")
