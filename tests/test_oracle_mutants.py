"""Planted mistakes in the oracle must be caught by its pins (CPU only).

Each case copies ``oracle/rmsnorm_oracle.c`` to a temporary directory, plants
one plausible slip by text substitution, compiles it with the oracle's own
flags, loads a private instance of the ``oracle`` package bound to the mutant
library, and runs every pin from ``tests/oracle_pins.py`` against it. At least
one pin must fail; the committed oracle itself is never modified.
"""
import importlib.util
import os
import subprocess

import pytest

import oracle
from tests import oracle_pins

MUTANTS = {
    "eps_outside_sqrt": ("double rms = sqrt(ms + e);", "double rms = sqrt(ms) + e;"),
    "sum_not_mean": ("double ms = ss / (double)H;", "double ms = ss;"),
    "mean_over_H_minus_1": ("double ms = ss / (double)H;", "double ms = ss / (double)(H - 1);"),
    "abs_not_square": ("ss += v[i] * v[i];", "ss += fabs(v[i]);"),
    "weight_dropped": ("y[i] = v[i] / rms * wi;", "y[i] = v[i] / rms;"),
    "weight_wrong_index": ("double wi = w ? load16(w, i, dtype) : 1.0;",
                           "double wi = w ? load16(w, H - 1 - i, dtype) : 1.0;"),
    "normalise_unrounded_sum": ("row[i] = load16(&rb, 0, dtype); /* normalise the stored residual */",
                                "row[i] = s;"),
    "residual_not_written_rounded": ("r_out[t * H + i] = rb;\n            row[i] = load16(&rb, 0, dtype); /* normalise",
                                     "r_out[t * H + i] = store16(load16(x, t * H + i, dtype), dtype);\n            row[i] = load16(&rb, 0, dtype); /* normalise"),
    "scale_inverted": ("double s = amax / 448.0;", "double s = 448.0 / amax;"),
    "fp8_max_240": ("oracle_f64_to_e4m3_satfinite(448.0 * p / pmax)",
                    "oracle_f64_to_e4m3_satfinite(240.0 * p / pmax)"),
    "ties_away_from_zero": ("r = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0; /* tie: to even */",
                            "r = fl + 1.0;"),
    "no_subnormals": ("if (E < emin) E = emin; /* subnormal range: fixed quantum */",
                      "if (E < emin) return 0.0;"),
    "f16_sign_dropped": ("    return sign ? -v : v;\n}\n\ndouble oracle_e4m3_to_f64",
                         "    return v;\n}\n\ndouble oracle_e4m3_to_f64"),
    "e4m3_bias_off_by_one": ("v = ldexp((double)(8 + m), e - 10);", "v = ldexp((double)(8 + m), e - 11);"),
    "e4m3_no_saturation": ("if (r > 448.0) r = 448.0;", "if (r > 480.0) r = 480.0;"),
    "swiglu_sign_of_exponent": ("double y = a / (1.0 + exp(-a)) * b;",
                                "double y = a / (1.0 + exp(a)) * b;"),
    "swiglu_halves_swapped": ("double y = a / (1.0 + exp(-a)) * b;",
                              "double y = b / (1.0 + exp(-b)) * a;"),
    "swiglu_no_gate_in_numerator": ("double y = a / (1.0 + exp(-a)) * b;",
                                    "double y = 1.0 / (1.0 + exp(-a)) * b;"),
    "swiglu_scale_240": ("double s = amax / 448.0;\n        scale[t] = (float)s;\n        for (int64_t i = 0; i < I; ++i) {",
                         "double s = amax / 240.0;\n        scale[t] = (float)s;\n        for (int64_t i = 0; i < I; ++i) {"),
    "gemm_b_transposed": ("const uint8_t* b = B + n * K;", "const uint8_t* b = B + n;"),
    "gemm_a_scale_dropped": ("double y = acc * (double)a_scale[m] * (double)b_scale[n];",
                             "double y = acc * (double)b_scale[n];"),
    "gemm_scales_swapped": ("double y = acc * (double)a_scale[m] * (double)b_scale[n];",
                            "double y = acc * (double)a_scale[n % M] * (double)b_scale[m % N];"),
    "allreduce_sticky_dropped": ("if (sticky) top |= 1;", "if (0) top |= 1;"),
    "allreduce_sign_ignored": ("acc_add(&acc, v < 0, m, (k - 24) - ACC_LSB);",
                               "acc_add(&acc, 0, m, (k - 24) - ACC_LSB);"),
    "allreduce_last_rank_dropped": ("for (int r = 0; r < W; ++r) {\n            double v = load16(parts",
                                    "for (int r = 0; r < W - 1; ++r) {\n            double v = load16(parts"),
    "allreduce_zero_sign": ("if (s == 0.0) s = all_neg_zero ? -0.0 : 0.0;", "if (s == 0.0) s = 0.0;"),
    "allreduce_inf_minus_inf": ("if (nan || (pinf && ninf)) s = NAN;", "if (nan) s = NAN;"),
    "allreduce_in_binary64": ("            s = acc_to_f64_odd(&acc);",
                              "            s = 0.0;\n            for (int r = 0; r < W; ++r) s += load16(parts + (int64_t)r * n, i, dtype);"),
    "allreduce_carry_lost": ("        carry = c1 | c2;", "        carry = c1;"),
    "bf16_overflow_threshold": ("if (r > maxf) return sign | 0x7f80; /* overflow to infinity */",
                                "if (r >= maxf) return sign | 0x7f80;"),
}


def _mutant_module(tmp_path, name, old, new):
    src = open(oracle._SRC).read()
    assert src.count(old) >= 1, f"mutation {name!r} no longer applies"
    mutated = src.replace(old, new)
    c = tmp_path / f"{name}.c"
    c.write_text(mutated)
    so = tmp_path / f"lib{name}.so"
    subprocess.check_call(["gcc", *oracle.CFLAGS, str(c), "-o", str(so), "-lm"])
    spec = importlib.util.spec_from_file_location(
        f"oracle_mutant_{name}", os.path.join(os.path.dirname(oracle._SRC), "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod._SRC, mod._LIB = str(c), str(so)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path, golden):
    old, new = MUTANTS[name]
    mod = _mutant_module(tmp_path, name, old, new)
    caught = []
    for pin in oracle_pins.PINS:
        try:
            pin(mod, golden)
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {name!r}"
