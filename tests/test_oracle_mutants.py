"""Planted mistakes in copies of the oracle must each be caught by some pin.

Each mutant is a one-token textual change of oracle/delta_rule_oracle.c that a
plausible implementation slip would produce (a flipped sign, a dropped term, a
wrong index, a transposed operand).  The copy is compiled into a temporary
directory; the real oracle is never modified.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "delta_rule_oracle.c")

# (name, original text, replacement, occurrence index to replace)
MUTANTS = [
    ("erase_sign", "e[j] = vt[j] - pred;", "e[j] = vt[j] + pred;", 0),
    ("write_missing_beta", "u[j] = bt * e[j];", "u[j] = e[j];", 0),
    ("kda_gate_channel_index", "return exp(J->loga[row_k(J, b, t, h) + c]);",
     "return exp(J->loga[row_k(J, b, t, h)]);", 0),
    ("gdn_gate_off_by_one_token", "if (J->variant == ORACLE_GATED) return exp(J->loga[row_s(J, b, t, h)]);",
     "if (J->variant == ORACLE_GATED) return exp(J->loga[row_s(J, b, t > 0 ? t - 1 : 0, h)]);", 0),
    ("output_query_reversed", "for (int c = 0; c < DK; ++c) acc += S[c * DV + j] * qt[c];",
     "for (int c = 0; c < DK; ++c) acc += S[c * DV + j] * qt[DK - 1 - c];", 0),
    ("write_outer_transposed", "for (int j = 0; j < DV; ++j) S[c * DV + j] += kt[c] * u[j];",
     "for (int j = 0; j < DV; ++j) S[c * DV + j] += kt[j % DK] * u[c % DV];", 0),
    ("bwd_dSp_sign", "dSp[c * DV + j] = G[c * DV + j] - bt * kt[c] * dU[j];",
     "dSp[c * DV + j] = G[c * DV + j] + bt * kt[c] * dU[j];", 0),
    ("bwd_no_decay_in_adjoint", "G[c * DV + j] = a * dSp[c * DV + j];", "G[c * DV + j] = dSp[c * DV + j];", 0),
    ("bwd_dk_missing_erase_term", "acc += G[c * DV + j] * ut[j] - bt * Sp[c * DV + j] * dU[j];",
     "acc += G[c * DV + j] * ut[j];", 0),
    ("bwd_dq_from_prev_state", "if (dOt)\n                        for (int j = 0; j < DV; ++j) acc += St[c * DV + j] * dOt[j];",
     "if (dOt)\n                        for (int j = 0; j < DV; ++j) acc += Sp[c * DV + j] * dOt[j];", 0),
    ("bwd_dbeta_uses_u", "for (int j = 0; j < DV; ++j) acc += et[j] * dU[j];",
     "for (int j = 0; j < DV; ++j) acc += ut[j] * dU[j];", 0),
    ("bwd_gate_grad_wrong_state", "acc += dSp[c * DV + j] * Sp[c * DV + j];",
     "acc += dSp[c * DV + j] * St[c * DV + j];", 0),
    ("chunk_decay_sign", "a += kr[c] * ki[c] * exp(g[r * DK + c] - g[i * DK + c]);",
     "a += kr[c] * ki[c] * exp(g[i * DK + c] - g[r * DK + c]);", 0),
    ("chunk_no_state_decay", "double acc = exp(gl) * S[c * DV + j];", "double acc = S[c * DV + j];", 0),
    ("chunk_causal_diag_dropped", "for (int i = 0; i <= r; ++i) {", "for (int i = 0; i < r; ++i) {", 0),
    ("chunk_A_includes_diagonal", "if (i < r) {", "if (i <= r) {", 0),
]


def _mutant_lib(tmp_path, name, old, new, occ):
    src = open(SRC).read()
    parts = src.split(old)
    assert len(parts) > occ + 1, f"mutation site for {name} not found"
    mutated = old.join(parts[:occ + 1]) + new + old.join(parts[occ + 1:])
    assert mutated != src
    c = tmp_path / f"{name}.c"
    c.write_text(mutated)
    so = tmp_path / f"lib{name}.so"
    subprocess.check_call(["gcc", "-O1", "-std=c99", "-D_POSIX_C_SOURCE=200809L", "-fPIC", "-shared", "-o", str(so),
                           str(c), "-lm", "-lpthread"])
    return oracle.load_library(str(so))


@pytest.mark.parametrize("name,old,new,occ", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new, occ):
    lib = _mutant_lib(tmp_path, name, old, new, occ)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, RuntimeError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutant {name}"
