"""The pins must be strong enough to catch plausible mistakes in the oracle.

Each case below copies oracle/ssm_oracle.c, plants one mistake by text
substitution (in every copy of the line), builds the copy on the CPU and runs
every pin of test_oracle_pins.py, test_oracle_complex_pins.py and
test_oracle_mimo_pins.py against it: at
least one pin has to fail.
"""
import os
import shutil

import pytest

import oracle
from oracle import build as oracle_build
from tests import test_oracle_complex_pins as complex_pins
from tests import test_oracle_mimo_pins as mimo_pins
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "ssm_oracle.c")

MUTANTS = {
    "drop_skip_term": ("acc += D_d * x;", "(void)D_d;"),
    "output_uses_previous_state": ("h[n] = abar * h[n] + bbar * x;    /* h_t = Abar h_{t-1} + Bbar x_t */\n"
                                   "            acc += Ct[n] * h[n];",
                                   "acc += Ct[n] * h[n];\n            h[n] = abar * h[n] + bbar * x;"),
    "decay_sign_flipped": ("*abar = exp(z);", "*abar = exp(-z);"),
    "euler_input_matrix": ("*bbar = phi * delta * b;", "*bbar = delta * b;"),
    "input_matrix_missing_delta": ("*bbar = phi * delta * b;", "*bbar = phi * b;"),
    "b_and_c_swapped": ("const double *Bt = B + t * nstate;\n        const double *Ct = C + t * nstate;",
                        "const double *Bt = C + t * nstate;\n        const double *Ct = B + t * nstate;"),
    "state_not_reset_per_row": ("h[n] = h0 ? h0[(b * channels + d) * nstate + n] : 0.0;",
                                "h[n] = h0 ? h0[(b * channels + d) * nstate + n] : (r == 0 ? 0.0 : h[n]);"),
    "token_stride_ignored": ("double x = u[t * stride];", "double x = u[t];"),
    "a_row_of_wrong_channel": ("A + d * nstate, ", "A + ((d + 1) % channels) * nstate, "),
    "b_uses_wrong_batch": ("len ? B + (size_t)(b * len) * (size_t)nstate : NULL,",
                           "len ? B : NULL,"),
    "expm1_replaced_by_exp": ("expm1(z) / z", "exp(z) / z"),
    # the exponential-Euler and trapezoidal options
    "euler_input_missing_delta": ("input = dt * Bt[n] * x;", "input = Bt[n] * x;"),
    "trapezoid_previous_not_decayed": ("previous = abar * B[(t - 1) * nstate + n] * u[(t - 1) * stride];",
                                       "previous = B[(t - 1) * nstate + n] * u[(t - 1) * stride];"),
    "trapezoid_full_weights": ("input = 0.5 * dt * (previous + Bt[n] * x);", "input = dt * (previous + Bt[n] * x);"),
    "trapezoid_previous_is_current_x": ("abar * B[(t - 1) * nstate + n] * u[(t - 1) * stride]",
                                        "abar * B[(t - 1) * nstate + n] * u[t * stride]"),
    "methods_decay_sign_flipped": ("double abar = exp(dt * A_row[n]);", "double abar = exp(-dt * A_row[n]);"),
    # the backward
    "backward_adjoint_not_decayed": ("lam[n] *= r;", "(void)r;"),
    "backward_dc_from_previous_state": ("dC[k * nstate + n] += g * ht;", "dC[k * nstate + n] += g * hprev;"),
    "backward_psi_sign": ("return (z * exp(z) - expm1(z)) / (z * z);", "return (z * exp(z) + expm1(z)) / (z * z);"),
    "backward_psi_series_coefficient": ("1.0 / 8.0 + z / 30.0", "1.0 / 6.0 + z / 30.0"),
    "backward_psi_series_cubic_term": ("1.0 / 8.0 + z / 30.0", "1.0 / 8.0 + z / 24.0"),
    "backward_psi_series_range": ("if (fabs(z) < 1e-3)", "if (fabs(z) < 1e-1)"),
    "backward_db_missing_x": ("dB[k * nstate + n] += lam[n] * x * phi * dt;", "dB[k * nstate + n] += lam[n] * phi * dt;"),
    "backward_ddelta_missing_a": ("ddt += lam[n] * r * (a * hprev + bn * x);", "ddt += lam[n] * r * (hprev + bn * x);"),
    "backward_adjoint_before_output": ("lam[n] += C[k * nstate + n] * g;           /* lam_t                       */",
                                       "(void)0;"),
    # the complex-valued state
    "complex_output_from_imaginary_part": ("acc += Ct[n] * creal(h[n]);", "acc += Ct[n] * cimag(h[n]);"),
    "complex_rotation_sign": ("double complex a = Are_row[n] + I * Aim_row[n];",
                              "double complex a = Are_row[n] - I * Aim_row[n];"),
    "complex_input_missing_division": ("(abar - 1.0) / z;", "(abar - 1.0);"),
    "complex_rotation_dropped": ("double complex abar = cexp(z);", "double complex abar = exp(creal(z));"),
    "complex_state_layout_swapped": ("h[n] = s0 ? s0[0] + I * s0[1] : 0.0;", "h[n] = s0 ? s0[1] + I * s0[0] : 0.0;"),
    # the multi-input multi-output state
    "mimo_input_sum_keeps_last_rank": ("in += bbar * xt[r * channels];", "in = bbar * xt[r * channels];"),
    "mimo_output_gate_shared": ("acc += Ct[r * nstate + n] * h[n];", "acc += Ct[n] * h[n];"),
    "mimo_input_column_mismatched": ("zoh_discretise(dt, A_row[n], Bt[r * nstate + n], &abar, &bbar);",
                                     "zoh_discretise(dt, A_row[n], Bt[((r + 1) % ranks) * nstate + n], &abar, &bbar);"),
    "mimo_skip_from_first_input": ("acc += D_d * xt[r * channels];", "acc += D_d * xt[0];"),
    "mimo_input_rank_stride": ("in += bbar * xt[r * channels];", "in += bbar * xt[r];"),
    "mimo_output_rank_layout": ("y[(t * ranks + r) * channels] = acc;", "y[(r * len + t) * channels] = acc;"),
}

def _pin_calls(module):
    """Every (name, function, keyword arguments) a pin module's tests run
    with: parametrized pins are expanded over their parameter values."""
    calls = []
    for name in sorted(dir(module)):
        if not name.startswith("test_"):
            continue
        fn = getattr(module, name)
        combos = [{}]
        for mark in getattr(fn, "pytestmark", []):
            if mark.name != "parametrize":
                continue
            argnames, values = mark.args[0], mark.args[1]
            keys = [k.strip() for k in argnames.split(",")] if isinstance(argnames, str) else list(argnames)
            rows = [v if len(keys) > 1 else (v,) for v in values]
            combos = [dict(c, **dict(zip(keys, r))) for c in combos for r in rows]
        for kw in combos:
            calls.append((name, fn, kw))
    return calls


PIN_CALLS = _pin_calls(pins) + _pin_calls(complex_pins) + _pin_calls(mimo_pins)


def test_every_pin_call_binds():
    """The harness calls each pin with the oracle and its parameters only; a
    call that cannot bind would count as a catch for every mutant."""
    import inspect
    for name, fn, kw in PIN_CALLS:
        inspect.signature(fn).bind(None, **kw)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    # a line that both row loops (zero-order hold and the other discretisations)
    # contain is mutated in both
    assert text.count(old) >= 1, f"mutation anchor for {name} not found"
    src = tmp_path / "mutant.c"
    src.write_text(text.replace(old, new))
    lib = oracle_build.build(str(src), str(tmp_path / "libmutant.so"), force=True)
    mutant = oracle.Oracle(lib)
    failed = []
    for pin_name, test, kw in PIN_CALLS:
        try:
            test(mutant, **kw)
        except Exception:          # an assertion or a shape/NaN failure both count
            failed.append(pin_name)
    assert failed, f"no pin caught mutant {name}"
    shutil.rmtree(tmp_path, ignore_errors=True)
