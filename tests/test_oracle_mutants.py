"""The pins have teeth: plausible mistakes planted in a copy of the oracle's C
source (a dropped term, a wrong sign, a wrong operand, a transposed index, a
wrong range, a wrong boundary) each make at least one pin fail.  CPU only; the
real oracle file is never modified."""
import os

import pytest

import oracle
from pins import ALL_PINS

# (name, text in ckda_oracle.c, replacement)
MUTANTS = [
    ("write_without_beta", "+= beta * k[i] * (v[j] - p[j])", "+= k[i] * (v[j] - p[j])"),
    ("write_sign_flipped", "+= beta * k[i] * (v[j] - p[j])", "-= beta * k[i] * (v[j] - p[j])"),
    ("erase_term_dropped", "+= beta * k[i] * (v[j] - p[j])", "+= beta * k[i] * (v[j])"),
    ("erase_reads_with_q", "acc += k[i] * S[(size_t)i * dv + j];", "acc += q[i] * S[(size_t)i * dv + j];"),
    ("gate_not_applied", "for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= alpha[i];",
     "for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= 1.0;"),
    ("ckda_gate_unsigned", "alpha[i] = 2.0 * sigmoid(a[i]) - 1.0;", "alpha[i] = sigmoid(a[i]);"),
    ("ckda_beta_unextended", "*beta = 2.0 * sigmoid(b);", "*beta = sigmoid(b);"),
    ("transition_gate_on_rows", "- beta * k[i] * k[j]) * alpha[j];", "- beta * k[i] * k[j]) * alpha[i];"),
    ("explicit_A_transposed", "acc += A[(size_t)i * dk + m] * S[(size_t)m * dv + j];",
     "acc += A[(size_t)m * dk + i] * S[(size_t)m * dv + j];"),
    ("initial_state_ignored", "if (J->S0)\n        memcpy", "if (0)\n        memcpy"),
    ("varlen_start_shifted", "t0 = J->cu[n];", "t0 = J->cu[n] + (n > 0);"),
    ("readout_uses_k", "acc += q[i] * S[(size_t)i * dv + j];\n            o[j]", "acc += k[i] * S[(size_t)i * dv + j];\n            o[j]"),
    # backward
    ("bwd_readout_grad_uses_k", "dS[(size_t)i * dv + j] += q[i] * dO[j];",
     "dS[(size_t)i * dv + j] += k[i] * dO[j];"),
    ("bwd_dq_from_previous_state", "acc += S_cur[(size_t)i * dv + j] * dO[j];",
     "acc += S_prev[(size_t)i * dv + j] * dO[j];"),
    ("bwd_erase_adjoint_dropped", "dS[(size_t)i * dv + j] += k[i] * (-beta * du[j]);",
     "dS[(size_t)i * dv + j] += 0.0 * k[i] * (-beta * du[j]);"),
    ("bwd_dp_sign_flipped", "acc += St[(size_t)i * dv + j] * (-beta * du[j]);",
     "acc += St[(size_t)i * dv + j] * (beta * du[j]);"),
    ("bwd_dbeta_without_erase", "dbeta += acc * (v[j] - p[j]);", "dbeta += acc * v[j];"),
    ("bwd_dalpha_from_new_state", "acc += dS[(size_t)i * dv + j] * S_prev[(size_t)i * dv + j];",
     "acc += dS[(size_t)i * dv + j] * S_cur[(size_t)i * dv + j];"),
    ("bwd_state_grad_ungated", "for (int j = 0; j < dv; ++j) dS[(size_t)i * dv + j] *= alpha[i];",
     "for (int j = 0; j < dv; ++j) dS[(size_t)i * dv + j] *= 1.0;"),
    ("bwd_ckda_derivative_halved", "(af == 1 ? 2.0 * sigmoid_deriv(a[i]) : 1.0)",
     "(af == 1 ? sigmoid_deriv(a[i]) : 1.0)"),
    ("bwd_checkpoint_off_by_one", "memcpy(states, ckpt + (size_t)sg * dd",
     "memcpy(states, ckpt + (size_t)(sg > 0 ? sg - 1 : 0) * dd"),
    # DeltaProduct form
    ("product_second_update_skipped", "for (int j = 0; j < nh; ++j) {",
     "for (int j = 0; j < 1; ++j) {"),
    ("product_gate_twice", "for (int c = 0; c < dv; ++c) S[(size_t)i * dv + c] *= alpha[i];",
     "for (int c = 0; c < dv; ++c) S[(size_t)i * dv + c] *= alpha[i] * alpha[i];"),
    ("product_readout_sign", "o[row * dv + c] = acc;", "o[row * dv + c] = -acc;"),
    ("product_strength_of_first_update", "gate_values(NULL, b[sub], 0,",
     "gate_values(NULL, b[((size_t)(tok0 + t) * nh) * H + h], 0,"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    src = open(oracle.SOURCE).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new, 1))
    so = oracle.compile_c(str(path), str(tmp_path / f"lib{name}.so"))
    mutant = oracle.Oracle(so)
    failed = []
    for pin in ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError, FloatingPointError):
            failed.append(pin.__name__)
    assert failed, f"no pin catches the planted mistake '{name}'"
