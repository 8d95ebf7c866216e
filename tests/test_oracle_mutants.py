"""Planted mistakes in the oracle must be caught by its pins.

Each mutant is a copy of oracle/oracle.c with one plausible error (a dropped
term or clamp, a wrong comparison, a transposed operand, a wrong decode, a wrong
quantization rule or scale); it is
compiled on the CPU into a temporary library, swapped in for the real one, and
the pin tests of test_oracle_pins.py are run against it.  Every mutant must
fail at least one pin.  Nothing here touches a GPU.
"""
import ctypes
import importlib.util
import os
import subprocess
import tempfile

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "oracle", "oracle.c")

MUTANTS = {
    "hidden_relu_dropped": ("h[j] = u > 0.0 ? u : 0.0;", "h[j] = u;"),
    "tie_counts_active": ("mask[i] = z[i] > 0.0 ? 1 : 0;", "mask[i] = z[i] >= 0.0 ? 1 : 0;"),
    "B_transposed": ("ld(B, dt, (size_t)j * n + i)", "ld(B, dt, (size_t)i * r + j)"),
    "A_transposed": ("ld(A, dt, (size_t)k * r + j)", "ld(A, dt, (size_t)j * d + k)"),
    "predictor_bias_dropped": ("z[i] = s + ld(c, dt, i);", "z[i] = s;"),
    "relu_bias_dropped": ("double g = up + ld(bias, dt, i);", "double g = up;"),
    "reglu_gate_clamp_dropped": ("a[i] = (g > 0.0 ? g : 0.0) * up;", "a[i] = g * up;"),
    "down_transposed": ("ld(w_down, dt, (size_t)j * n + list[t])", "ld(w_down, dt, (size_t)list[t] * d + j)"),
    "half_exponent_off": ("expo - 25", "expo - 24"),
    "half_sign_dropped": ("return sign ? -v : v;", "return v;"),
    "inactive_not_skipped": ("if (!mask[i]) {\n            a[i] = 0.0;\n            continue;\n        }\n        double up = 0.0;\n"
                             "        for (int32_t k = 0; k < d; ++k) up += ld(w_up,",
                             "if (0 && !mask[i]) {\n            a[i] = 0.0;\n            continue;\n        }\n"
                             "        double up = 0.0;\n        for (int32_t k = 0; k < d; ++k) up += ld(w_up,"),
    "down_coefficient_by_position": ("s += a[list[t]] *", "s += a[t] *"),
    "reglu_gate_bias_dropped": ("g += ld(bias, dt, i);", "g += 0.0;"),
    "preact_bias_dropped": ("g[i] = s + ld(bias, dt, i);", "g[i] = s;"),
    # int8 rows
    "quant_scale_by_qmax_plus_1": ("const float s = amax / (float)qmax;", "const float s = amax / (float)(qmax + 1);"),
    "quant_round_half_away": ("c = (int32_t)rintf(v / s);", "c = (int32_t)roundf(v / s);"),
    "quant_truncates": ("c = (int32_t)rintf(v / s);", "c = (int32_t)(v / s);"),
    "q_down_scale_of_up": ("* (double)s_down[i]);", "* (double)s_up[i]);"),
    "q_relu_bias_dropped": ("const double pre = up + ld(bias, dt, i);", "const double pre = up;"),
    "q_gate_clamp_dropped": ("a[i] = (gate > 0.0 ? gate : 0.0) * up;", "a[i] = gate * up;"),
    "q_inactive_not_skipped": ("if (!mask[i]) {\n            a[i] = 0.0;\n            continue;\n        }\n        double up = 0.0;\n"
                               "        for (int32_t k = 0; k < d; ++k) up += ((double)q_up",
                               "if (0 && !mask[i]) {\n            a[i] = 0.0;\n            continue;\n        }\n"
                               "        double up = 0.0;\n        for (int32_t k = 0; k < d; ++k) up += ((double)q_up"),
    "q_gate_scale_dropped": ("((double)q_gate[(size_t)i * d + k] * (double)s_gate[i])", "((double)q_gate[(size_t)i * d + k])"),
}


def _pins_module():
    spec = importlib.util.spec_from_file_location("_pins", os.path.join(HERE, "test_oracle_pins.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _pin_calls(pins):
    import numpy as np
    calls = [pins.test_half_decode_all_bit_patterns, pins.test_golden_stack_two_layers,
             pins.test_predictor_against_sigmoid_definition, pins.test_tie_and_nan_are_inactive,
             pins.test_single_active_neuron_closed_form, pins.test_empty_set_gives_zero]
    for dt in (np.float16, np.float32):
        calls.append(lambda dt=dt: pins.test_golden_powerinfer_relu(dt))
        calls.append(lambda dt=dt: pins.test_golden_powerinfer_reglu(dt))
        for act in ("relu", "reglu"):
            calls.append(lambda dt=dt, act=act: pins.test_exact_set_equals_dense(act, dt))
    for act in ("relu", "reglu"):
        calls.append(lambda act=act: pins.test_all_ones_mask_equals_dense(act))
        for bits in (8, 4):
            calls.append(lambda act=act, bits=bits: pins.test_forward_q_equals_forward_on_an_exact_grid(act, bits))
    calls += [pins.test_quantizer_hand_values, pins.test_quantizer_hand_values_int4, pins.test_lookahead_hand_example]
    for bits in (8, 4):
        calls.append(lambda bits=bits: pins.test_quantizer_invariants(bits))
    return calls


def _compile(src_text, tmpdir, name):
    c_path = os.path.join(tmpdir, f"{name}.c")
    so_path = os.path.join(tmpdir, f"lib{name}.so")
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O1", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared", "-std=c99",
                    c_path, "-o", so_path, "-lm"], check=True)
    return so_path


def _bind(path):
    """A CDLL with the same signatures the oracle module sets on its own library."""
    saved = oracle._lib
    try:
        oracle._lib = None
        real = oracle._load()
        lib = ctypes.CDLL(path)
        for fn in ("oracle_decode", "oracle_predictor", "oracle_preact", "oracle_ffn_masked",
                   "oracle_forward", "oracle_max_threads", "oracle_quantize", "oracle_ffn_masked_q"):
            getattr(lib, fn).argtypes = getattr(real, fn).argtypes
            getattr(lib, fn).restype = getattr(real, fn).restype
        return lib
    finally:
        oracle._lib = saved


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    src = open(SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    pins = _pins_module()
    with tempfile.TemporaryDirectory() as tmp:
        lib = _bind(_compile(src.replace(old, new), tmp, name))
        saved = oracle._lib
        oracle._lib = lib
        failures = 0
        try:
            for call in _pin_calls(pins):
                try:
                    call()
                except AssertionError:
                    failures += 1
        finally:
            oracle._lib = saved
    assert failures > 0, f"no pin caught mutant {name}"


# The look-ahead stack and the code widths are bookkeeping in oracle/__init__.py: their
# mutants are copies of that module with one mistake, loaded beside the real one (same
# compiled library).
PY_SRC = os.path.join(os.path.dirname(HERE), "oracle", "__init__.py")
PY_MUTANTS = {
    "lookahead_from_current_input": ('xpred = xin if li == 0 else records[li - 1]["x_in"]', "xpred = xin"),
    "lookahead_residual_dropped": ("""        records.append(dict(x_in=xin, x_pred=xpred, z=z, mask=mask, y=y, mismatches=mismatches))
        resid = resid + y""", """        records.append(dict(x_in=xin, x_pred=xpred, z=z, mask=mask, y=y, mismatches=mismatches))
        resid = y"""),
    "int4_qmax_8": ("QMAX = {8: 127, 4: 7}", "QMAX = {8: 127, 4: 8}"),
    "lookahead_input_not_rounded": ("""        xin = resid.astype(dt)  # round to nearest even
        xpred = xin if""", """        xin = resid.copy()
        xpred = xin if"""),
}


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_python_mutant_is_caught(name):
    src = open(PY_SRC).read()
    old, new = PY_MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    spec = importlib.util.spec_from_loader("_oracle_mutant", loader=None)
    mod = importlib.util.module_from_spec(spec)
    mod.__file__ = PY_SRC
    exec(compile(src.replace(old, new), PY_SRC, "exec"), mod.__dict__)
    mod._lib = oracle._load()
    pins = _pins_module()
    pins.oracle = mod
    failures = 0
    for call in (pins.test_lookahead_hand_example, lambda: pins.test_lookahead_special_cases_equal_the_stack("relu"),
                 pins.test_quantizer_hand_values_int4):
        try:
            call()
        except AssertionError:
            failures += 1
    assert failures > 0, f"no pin caught mutant {name}"


def test_unmutated_passes_every_pin():
    pins = _pins_module()
    for call in _pin_calls(pins):
        call()
