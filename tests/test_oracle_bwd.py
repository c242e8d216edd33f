"""The oracle's backward pass against its pins, and planted mistakes in it caught (CPU)."""
import pytest

import oracle
import oracle_bwd_pins


@pytest.mark.parametrize("pin", oracle_bwd_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_bwd_pin(pin):
    pin(oracle.load())


# Each a plausible slip in the reverse sweep: a dropped term, a wrong sign, the state on the
# wrong side of the write, a wrong gate derivative.  One exact substitution each.
MUTANTS = {
    "dk_drops_state_term": ("dk[t * dk_ + i] = -at * (gr + sg) + da * dadl * 2.0 * kx[i];",
                            "dk[t * dk_ + i] = -at * gr + da * dadl * 2.0 * kx[i];"),
    "dk_drops_gate_term": ("dk[t * dk_ + i] = -at * (gr + sg) + da * dadl * 2.0 * kx[i];",
                           "dk[t * dk_ + i] = -at * (gr + sg);"),
    "dq_before_write": ("acc += Sc[i * dv_ + j] * dox[j];", "acc += Sp[i * dv_ + j] * dox[j];"),
    "state_gradient_sign": ("G[i * dv_ + j] -= at * kx[i] * g[j];", "G[i * dv_ + j] += at * kx[i] * g[j];"),
    "dalpha_sign": ("da -= g[j] * r[j];", "da += g[j] * r[j];"),
    "dbeta_euler_factor": ("dadb = exp(-beta[t] * l2);", "dadb = 1.0;"),
    "series_coefficient": ("x / 3.0", "x / 6.0"),
    "residual_without_value": ("double rj = -vx[j], gj = 0.0;", "double rj = 0.0, gj = 0.0;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_bwd_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    with open(oracle.SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation target for {name} not found exactly once"
    mut_src = tmp_path / "mutant.c"
    mut_src.write_text(src.replace(old, new))
    lib = oracle.load(oracle.build(str(mut_src), str(tmp_path / "mutant.so"), force=True))
    caught = []
    for pin in oracle_bwd_pins.ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {name!r}"
