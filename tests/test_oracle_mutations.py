"""Planted mistakes: each test copies the oracle's C source, plants one
plausible mistake (a dropped term, a wrong sign, index, divisor, rounding
or clamp), compiles the copy and runs the pins of test_oracle_pins.py against
it. At least one pin must fail for every mistake; the unchanged copy, built
the same way, must pass them all. CPU only; nothing here touches the CUDA
library."""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "ttq_oracle.c")
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")
OUT = os.path.join(ROOT, "_build", "oracle_variants")

# (name, text in the source, replacement): the first occurrence is replaced
MISTAKES = [
    ("statistic_of_x_not_abs_x",
     "double a = fabs((double)row[j]);", "double a = (double)row[j];"),
    ("mean_over_T_plus_one",
     "m[j] = sum[j] / (double)T_total;",
     "m[j] = sum[j] / (double)(T_total + 1);"),
    ("shrink_weights_swapped",
     "(1.0 - lambda) * m[j] + lambda * mbar",
     "lambda * m[j] + (1.0 - lambda) * mbar"),
    ("given_mean_replaced_by_own_statistic",
     "double c = (1.0 - lambda) * m + lambda * mbar;",
     "double c = (1.0 - lambda) * m + lambda * m;"),
    ("exponent_alpha_times_p",
     "sj = pow(c, alpha / p);", "sj = pow(c, alpha * p);"),
    ("range_not_widened_to_zero",
     "float mn = 0.0f, mx = 0.0f; /* the range always contains 0 */",
     "float mn = w[0], mx = w[0];"),
    ("no_zero_point",
     "float z = clampf(rintf(-mn / d), 0.0f, qmax);", "float z = 0.0f;"),
    ("round_half_away_from_zero",
     "float v = rintf(w[i] / d) + z;", "float v = roundf(w[i] / d) + z;"),
    ("quotient_by_rounded_reciprocal",
     "float v = rintf(w[i] / d) + z;",
     "float v = rintf(w[i] * (1.0f / d)) + z;"),
    ("zero_point_by_rounded_reciprocal",
     "float z = clampf(rintf(-mn / d), 0.0f, qmax);",
     "float z = clampf(rintf(-mn * (1.0f / d)), 0.0f, qmax);"),
    ("clamp_one_code_short",
     "q[i] = (uint8_t)clampf(v, 0.0f, qmax);",
     "q[i] = (uint8_t)clampf(v, 0.0f, qmax - 1.0f);"),
    ("adjacent_codes_swapped_in_packing",
     "int bit = c * bits;", "int bit = (c ^ 1) * bits;"),
    ("projection_without_inverse_scale",
     "xs[j] = (double)x[j] * (double)inv_s[j];", "xs[j] = (double)x[j];"),
    ("dequantization_without_zero_point",
     "acc += xs[j] * ((q - z) * (double)delta[n * G + j / group]);",
     "acc += xs[j] * (q * (double)delta[n * G + j / group]);"),
    ("low_rank_factor_transposed",
     "acc += u[rho] * (double)B[n * r + rho];",
     "acc += u[rho] * (double)B[rho * N + n];"),
    ("low_rank_term_on_scaled_x",
     "acc += (double)x[j] * (double)A[(int64_t)rho * K + j];",
     "acc += xs[j] * (double)A[(int64_t)rho * K + j];"),
    ("dequantized_weight_without_delta",
     "What_s[n * K + j] = (q - z) * (double)delta[n * G + j / group];",
     "What_s[n * K + j] = (q - z);"),
    ("loss_error_sign",
     "e[j] = (double)W[n * K + j] - W_eff[n * K + j];",
     "e[j] = (double)W[n * K + j] + W_eff[n * K + j];"),
    ("loss_not_divided_by_T",
     "return total / (double)T;", "return total;"),
    ("near_ties_never_counted",
     "int weight_tie = near_half(w[i] / d);", "int weight_tie = 0;"),
    ("near_ties_counted_two_steps_out",
     "return v == h || nextafterf(v, INFINITY) == h ||",
     "return v == h || nextafterf(nextafterf(v, INFINITY), INFINITY) == h ||"
     " nextafterf(nextafterf(v, -INFINITY), -INFINITY) == h ||"
     " nextafterf(v, INFINITY) == h ||"),
    ("zero_point_near_ties_ignored",
     "int zero_tie = near_half(-mn / d);", "int zero_tie = 0;"),
]


def build_variant(name, text):
    os.makedirs(OUT, exist_ok=True)
    c = os.path.join(OUT, f"{name}.c")
    so = os.path.join(OUT, f"{name}.so")
    with open(c, "w") as f:
        f.write(text)
    subprocess.check_call(["gcc", *oracle.CFLAGS, c, "-o", so, "-lm"])
    return so


def run_pins(lib):
    env = dict(os.environ, TTQ_ORACLE_LIB=lib)
    return subprocess.run(
        [sys.executable, "-m", "pytest", PINS, "-q", "-x", "-p",
         "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True,
        text=True, timeout=600)


def test_unchanged_copy_passes_the_pins():
    lib = build_variant("unchanged", open(SRC).read())
    r = run_pins(lib)
    assert r.returncode == 0, r.stdout[-3000:]


@pytest.mark.parametrize("name,old,new", MISTAKES,
                         ids=[m[0] for m in MISTAKES])
def test_each_planted_mistake_fails_a_pin(name, old, new):
    src = open(SRC).read()
    assert old in src, f"{name}: the planted text no longer occurs"
    lib = build_variant(name, src.replace(old, new, 1))
    r = run_pins(lib)
    # 1: a pin failed (not a crash, not a collection error)
    assert r.returncode == 1, f"{name}: exit {r.returncode}\n" + \
        r.stdout[-3000:]
