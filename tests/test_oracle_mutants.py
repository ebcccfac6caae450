"""The oracle's pins must catch plausible mistakes.

Each case copies the oracle source, plants one mistake (a dropped term, a wrong sign, a
swapped index, a transposed operand, a shifted tap, a missed reset), builds it on the CPU and
runs the pin suite against it: at least one pin has to fail.  Nothing here touches a GPU.
"""

import os
import shutil
import subprocess
import tempfile

import pytest

import oracle
from tests import test_backward_oracle as bwd_pins
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "rglru_oracle.c")

MUTANTS = {
    "transposed_gate_weights": ("widen(w_a, (long)i * dh + o, w_dtype)", "widen(w_a, (long)o * dh + i, w_dtype)"),
    "dropped_sqrt_normaliser": ("h[o] = a * h[o] + beta * (ig * xc[o]);", "h[o] = a * h[o] + (ig * xc[o]);"),
    "sign_of_log_decay": ("double log_a = c * r * log_a_base[o];", "double log_a = -c * r * log_a_base[o];"),
    "raw_x_instead_of_conv": ("h[o] = a * h[o] + beta * (ig * xc[o]);", "h[o] = a * h[o] + beta * (ig * widen(x, (long)t * ld + o, act_dtype));"),
    "tap_order_reversed": ("acc += (double)conv_w[k * conv_ld + j] * tail[k * tail_ld + j];", "acc += (double)conv_w[(2 - k) * conv_ld + j] * tail[k * tail_ld + j];"),
    "dropped_conv_bias": ("double acc = conv_b ? (double)conv_b[j] : 0.0;", "double acc = 0.0;"),
    "reset_keeps_state": ("for (int j = 0; j < dh; ++j) h[j] = 0.0;", "(void)0;"),
    "gate_bias_swapped": ("ga[o] = b_a ? (double)b_a[o] : 0.0;", "ga[o] = b_x ? (double)b_x[o] : 0.0;"),
    "input_gate_from_recurrence_weights": ("gx[o] += xi * widen(w_x, (long)i * dh + o, w_dtype);", "gx[o] += xi * widen(w_a, (long)i * dh + o, w_dtype);"),
    "gelu_tanh_by_default": ("    return 0.5 * v * erfc(-v / sqrt(2.0));", "    return 0.5 * v * (1.0 + tanh(0.7978845608028654 * (v + 0.044715 * v * v * v)));"),
    # constants of the tanh form perturbed within 1e-3 of the exact GeLU
    "gelu_tanh_constants": ("        return 0.5 * v * (1.0 + tanh(k * (v + 0.044715 * v * v * v)));",
                            "        return 0.5 * v * (1.0 + tanh(0.8 * (v + 0.0447 * v * v * v)));"),
}

PIN_TESTS = [
    pins.test_gelu_spot_values,
    pins.test_gelu_tanh_form_matches_torch,
    pins.test_closed_form_geometric_sum,
    pins.test_freeze_when_recurrence_gate_is_zero,
    pins.test_decay_strictly_inside_unit_interval,
    lambda: pins.test_bruteforce_unrolling_T8("f32"),
    pins.test_gate_orientation_is_in_major,
    pins.test_conv_identity_and_single_taps,
    pins.test_conv_matches_torch_conv1d_listing_form,
    pins.test_packed_rows_equal_separate_documents,
    pins.test_reset_cuts_all_dependence_on_the_past,
]


# Mistakes in the backward pass, each of which the backward pins must catch.
BACKWARD_MUTANTS = {
    "bwd_reset_keeps_gradient": ("g[o] = (reset && reset[t]) ? 0.0 : a * g[o];", "g[o] = a * g[o];"),
    "bwd_beta_term_sign": ("double q = dl_da * a * r - dl_dbeta * a * a * r_over_beta;",
                           "double q = dl_da * a * r + dl_dbeta * a * a * r_over_beta;"),
    "bwd_dropped_direct_input_path": ("dxc[e] = g[o] * beta * ig;", "dxc[e] = 0.0;"),
    "bwd_gelu_density_dropped": ("return 0.5 * erfc(-v / sqrt(2.0)) + v * exp(-0.5 * v * v) / sqrt(2.0 * pi);",
                                 "return 0.5 * erfc(-v / sqrt(2.0));"),
    "bwd_weight_grad_transposed": ("dw_a[(long)i * dh + o] += xct[i] * dga[o];",
                                   "dw_a[(long)o * dh + i] += xct[i] * dga[o];"),
    "bwd_conv_scatter_wrong_tap": ("if (src >= 0) dx[(long)src * ld + j] += (double)conv_w[k * conv_ld + j] * d;",
                                   "if (src >= 0) dx[(long)src * ld + j] += (double)conv_w[(3 - k) * conv_ld + j] * d;"),
    "bwd_gelu_tanh_chain_factor": ("k * (1.0 + 3.0 * 0.044715 * v * v);", "k * (1.0 + 0.044715 * v * v);"),
}

BACKWARD_PIN_TESTS = [
    bwd_pins.test_backward_matches_finite_differences,
    bwd_pins.test_gelu_tanh_derivative_matches_torch_autograd,
    bwd_pins.test_backward_frozen_state_closed_form,
    bwd_pins.test_backward_reset_at_the_first_token_cuts_the_initial_state,
    lambda: bwd_pins.test_gelu_derivative_matches_a_difference_quotient(0.7, 0),
]


def _build_mutant(old, new, tmp):
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor not found exactly once"
    path = os.path.join(tmp, "mutant.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib_path = os.path.join(tmp, "libmutant.so")
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC",
                           "-shared", "-o", lib_path, path, "-lm"])
    return lib_path


@pytest.mark.parametrize("name", sorted(BACKWARD_MUTANTS))
def test_backward_pins_catch_planted_mistake(name, monkeypatch):
    old, new = BACKWARD_MUTANTS[name]
    tmp = tempfile.mkdtemp(prefix="oracle_mutant_")
    try:
        monkeypatch.setattr(oracle, "_lib", oracle.load_library(_build_mutant(old, new, tmp)))
        caught = 0
        for pin in BACKWARD_PIN_TESTS:
            try:
                pin()
            except AssertionError:
                caught += 1
        assert caught >= 1, f"no backward pin caught the planted mistake {name}"
    finally:
        shutil.rmtree(tmp, ignore_errors=True)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    tmp = tempfile.mkdtemp(prefix="oracle_mutant_")
    try:
        path = os.path.join(tmp, "mutant.c")
        with open(path, "w") as f:
            f.write(src.replace(old, new))
        lib_path = os.path.join(tmp, "libmutant.so")
        subprocess.check_call(["gcc", "-O1", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC",
                               "-shared", "-o", lib_path, path, "-lm"])
        monkeypatch.setattr(oracle, "_lib", oracle.load_library(lib_path))
        failed = []
        for t in PIN_TESTS:
            try:
                t()
            except AssertionError:
                failed.append(getattr(t, "__name__", "bruteforce"))
        assert failed, f"no pin caught the planted mistake '{name}'"
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
