"""The oracle's gated flow against its pins, and planted mistakes in it (CPU only).

Each mutant is one exact text substitution in a copy of efla_oracle.c's gated recurrence:
the decay dropped, its sign flipped, applied to the write as well, the write gate abar
replaced by alpha, the decay's sign inside abar flipped.  Some gated pin must fail for each.
"""
import pytest

import oracle
import oracle_gated_pins


@pytest.mark.parametrize("pin", oracle_gated_pins.GATED_PINS, ids=lambda f: f.__name__)
def test_gated_pin(pin, oracle_lib):
    pin(oracle_lib)


MUTANTS = {
    "no_decay": ("const double dec = exp(g[t]);", "const double dec = 1.0;"),
    "decay_sign": ("const double dec = exp(g[t]);", "const double dec = exp(-g[t]);"),
    "decay_on_write": ("S[i * dv + j] = dec * (S[i * dv + j] - a * key[i] * m[j]) + ab * key[i] * value[j];",
                       "S[i * dv + j] = dec * (S[i * dv + j] - a * key[i] * m[j] + ab * key[i] * value[j]);"),
    "write_gate_is_alpha": ("ab = beta[t] * phi1(beta[t] * lambda - g[t]);", "ab = a;"),
    "write_gate_decay_sign": ("ab = beta[t] * phi1(beta[t] * lambda - g[t]);",
                              "ab = beta[t] * phi1(beta[t] * lambda + g[t]);"),
    "read_after_decay": ("m[j] += S[i * dv + j] * key[i];", "m[j] += exp(g[t]) * S[i * dv + j] * key[i];"),
    "initial_state_ignored": ("        if (S0 == NULL)\n            memset(", "        if (1)\n            memset("),
    "output_before_decay": ("out[j] += S[i * dv + j] * query[i];",
                            "out[j] += S[i * dv + j] * query[i] / exp(g[t]);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_gated_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    with open(oracle.SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation target for {name} not found exactly once"
    mut = tmp_path / "mutant.c"
    mut.write_text(src.replace(old, new))
    lib = oracle.load(oracle.build(str(mut), str(tmp_path / "mutant.so"), force=True))
    caught = []
    for pin in oracle_gated_pins.GATED_PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no gated pin catches the planted mistake {name!r}"
