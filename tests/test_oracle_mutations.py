"""Planted mistakes: every plausible error in the C oracle must fail some pin.

Each case copies oracle/mlstm_oracle.c to a temporary directory, applies one
textual mutation (a dropped term, a wrong sign, a wrong index or operand, a
wrong floor), builds it with gcc, points the oracle's loader at the mutant and
runs the pins of test_oracle_pins.py against it.  The committed oracle is never
modified.  A mutant that passes every pin means the pins are too weak.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

MUTATIONS = {
    "drop_input_gate": ("iprime * vt[r] * kt[c]", "vt[r] * kt[c]"),
    "logsigmoid_sign": ("- log1p(exp(-fabs(x)))", "+ log1p(exp(-fabs(x)))"),
    "floor_one_in_stabilised_units": ("fmax(fabs(nq), exp(-m))", "fmax(fabs(nq), 1.0)"),
    "forget_gate_drops_previous_m": ("fprime = exp(lf + m - m_new)", "fprime = exp(lf - m_new)"),
    "stabiliser_min_not_max": ("(lf + m > li) ? lf + m : li", "(lf + m < li) ? lf + m : li"),
    "readout_uses_k_not_q": ("acc += C[(size_t)r * dk + c] * qt[c]", "acc += C[(size_t)r * dk + c] * kt[c]"),
    "normaliser_drops_forget": ("n[c] = fprime * n[c] + iprime * kt[c]", "n[c] = n[c] + iprime * kt[c]"),
    "normaliser_no_abs": ("fmax(fabs(nq), exp(-m))", "fmax(nq, exp(-m))"),
    "gamma_wrong_exponent": ("ldexp(1.0, -5 - head)", "ldexp(1.0, -4 - head)"),
    "retention_gamma_per_block": ("head = bh % J->NH", "head = slice % J->NH"),
    "block_uses_wrong_key_slice": ("J->k + tok * J->DHQK + (size_t)blk * dk", "J->k + tok * J->DHQK"),
    "output_gate_ignored": ("J->og[tok * J->DHV + (size_t)blk * dv + r] : 1.0", "1.0 : 1.0"),
    "initial_m_ignored": ("if (J->m0) m = J->m0[bh];", ""),
    "update_uses_v_index_for_k": ("vt[r] * kt[c]", "vt[r] * kt[c % (dv < dk ? dv : dk)]"),
}

PIN_RUNS = [
    lambda: pins.test_sequential_equals_quadratic_parallel_form(1, False, False, (2, 3, 13, 6, 4)),
    lambda: pins.test_sequential_equals_quadratic_parallel_form(1, True, True, (1, 2, 17, 5, 7)),
    lambda: pins.test_sequential_equals_quadratic_parallel_form(2, True, False, (2, 2, 11, 8, 6)),
    lambda: pins.test_sequential_equals_quadratic_parallel_form(4, False, True, (1, 3, 9, 8, 12)),
    lambda: pins.test_retention_sequential_equals_parallel_form(True),
    lambda: pins.test_retention_geometric_series_closed_form(4),
    lambda: pins.test_retention_page_orientation_brute_force(),
    lambda: pins.test_retention_block_diagonal_uses_head_gamma(),
    lambda: pins.test_hand_derived_two_steps(),
    lambda: pins.test_unit_gates_reduce_to_floored_causal_linear_attention(),
    lambda: pins.test_stabiliser_does_not_change_h(2, True),
    lambda: pins.test_block_diagonal_equals_independent_subheads(),
]


def _build_mutant(tmp_path, old, new):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "mlstm_oracle.c")).read()
    assert src.count(old) >= 1, "mutation pattern not found: " + old
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O1", "-fPIC", "-shared", "-std=c11", "-pthread",
                           "-o", str(so), str(path), "-lm"])
    lib = ctypes.CDLL(str(so))
    lib.oracle_mlstm_sequential.argtypes = [ctypes.c_int] * 7 + [ctypes.c_void_p] * 13 + [ctypes.c_int]
    lib.oracle_mlstm_sequential.restype = ctypes.c_int
    return lib


def _pins_pass():
    for run in PIN_RUNS:
        try:
            run()
        except AssertionError:
            return False
    return True


def test_unmutated_oracle_passes_the_pin_subset():
    assert _pins_pass()


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutant_is_caught(name, tmp_path, monkeypatch):
    old, new = MUTATIONS[name]
    monkeypatch.setattr(oracle, "_lib", _build_mutant(tmp_path, old, new))
    assert not _pins_pass(), f"mutation {name!r} survived every pin"
