"""The oracle's pins catch plausible mistakes.

Each case below plants one mistake in a copy of oracle/kq_oracle.c (a wrong
sign, a dropped term, a transposed operand or index, an off-by-one, a wrong
rounding rule), builds the copy with the oracle's own flags, routes the oracle
module through it, and runs the pins of tests/test_oracle_pins.py against it.
At least one pin must fail for every mistake; the unmodified source must pass
them all.  The exhaustive E2M1 sweep is left out to keep this fast (the golden
grid and the random-pattern pins cover the E2M1 cases).
"""
from __future__ import annotations

import inspect
import itertools
import os

import pytest

from . import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "kq_oracle.c")

# name: (text in kq_oracle.c, replacement)
MUTANTS = {
    # LU factor [KQ Approach: unit-determinant LU factors]
    "U_corner_u_not_1_over_u": ("0.0, 1.0 / (double)u};", "0.0, (double)u};"),
    "L_entry_sign": ("{1.0, 0.0, (double)l, 1.0}", "{1.0, 0.0, -(double)l, 1.0}"),
    "inverse_as_Linv_Uinv": ("Fi[2 * r + c] = Ui[2 * r + 0] * Li[0 + c] + Ui[2 * r + 1] * Li[2 + c];",
                             "Fi[2 * r + c] = Li[2 * r + 0] * Ui[0 + c] + Li[2 * r + 1] * Ui[2 + c];"),
    # Kronecker product and its order
    "kron_inner_operand_transposed": ("B[(i % nbd) * nbd + (j % nbd)]", "B[(j % nbd) * nbd + (i % nbd)]"),
    "kron_order_reversed": ("kqo_kron(F[k], 2, acc, n, tmp);", "kqo_kron(acc, n, F[k], 2, tmp);"),
    "kron_order_reversed_n": ("kqo_kron(F, 2, acc, m, tmp);", "kqo_kron(acc, m, F, 2, tmp);"),
    "hadamard_H2_sign": ("{s, s, s, -s}", "{s, s, -s, s}"),
    # the transform y = x K
    "transform_transposed": ("(int64_t)i * KQO_N + j);", "(int64_t)j * KQO_N + i);"),
    "transform_first_term_dropped": ("for (int i = 0; i < KQO_N; i++) {\n          const double xi",
                                     "for (int i = 1; i < KQO_N; i++) {\n          const double xi"),
    "transform_n_transposed": ("(int64_t)i * n + j);", "(int64_t)j * n + i);"),
    # MXFP4: E8M0 scale, E2M1 codes, packing, non-finite blocks
    "e8m0_off_by_one": ("int e = (E - 1) - 2;", "int e = (E - 1) - 1;"),
    "e8m0_no_lower_clamp": ("if (e < -127) e = -127;", ""),
    "e2m1_ties_away_from_zero": ("&& (c & 1)) c++;", ") c++;"),
    "e2m1_sign_dropped": ("return c | (signbit(v) ? 8 : 0);", "return c;"),
    "e2m1_top_magnitude_5": ("{0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0}", "{0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 5.0}"),
    "pack_nibbles_swapped": ("(kqo_e2m1(v[2 * k]) | (kqo_e2m1(v[2 * k + 1]) << 4))",
                             "(kqo_e2m1(v[2 * k + 1]) | (kqo_e2m1(v[2 * k]) << 4))"),
    "amax_skips_element_0": ("for (int j = 0; j < KQO_N; j++) {\n        if (!isfinite(yb[j]))",
                             "for (int j = 1; j < KQO_N; j++) {\n        if (!isfinite(yb[j]))"),
    "nonfinite_block_byte_0": ("scales[r * nb + b] = 0xFF;", "scales[r * nb + b] = 0;"),
    "quantize_scale_inverted": ("ldexpf(1.0f, 127 - byte)", "ldexpf(1.0f, byte - 127)"),
    # bf16 rounding of the matrices, the comparison points, the inverse
    "bf16_ties_down": ("if (frac > 0.5 || (frac == 0.5 && fmod(lo, 2.0) != 0.0)) lo += 1.0;",
                       "if (frac > 0.5) lo += 1.0;"),
    "smooth_factor_dropped": ("(float)((double)f32_from_bf16(x[r * ldx + c]) * (double)inv_s[c])",
                              "(float)((double)f32_from_bf16(x[r * ldx + c]))"),
    "dequantize_scale_inverted": ("ldexp(1.0, byte - 127)", "ldexp(1.0, 127 - byte)"),
    "dequantize_inverse_transposed": ("(int64_t)j * KQO_N + i);", "(int64_t)i * KQO_N + j);"),
    # the W4A4 product
    # (a nibble swap on both operands leaves every dot product unchanged: not a mistake here)
    "mx_gemm_high_nibble_twice": ("const int code = (k & 1) ? (pair >> 4) : (pair & 0xF);\n  if (byte == 0xFF)",
                                  "const int code = (k & 1) ? (pair >> 4) : (pair >> 4);\n  if (byte == 0xFF)"),
    "mx_gemm_scale_of_next_block": ("scales[row * (K / KQO_N) + k / KQO_N];",
                                    "scales[row * (K / KQO_N) + (k / KQO_N + 1) % (K / KQO_N)];"),
    "mx_gemm_scale_sign": ("ldexp(kqo_e2m1_value(code), byte - 127)", "ldexp(kqo_e2m1_value(code), 127 - byte)"),
    "mx_gemm_last_element_dropped": ("for (int64_t k = 0; k < K; k++)\n        acc +=",
                                     "for (int64_t k = 0; k < K - 1; k++)\n        acc +="),
    # the AdaLN normalisation in front of the quantizer
    "adaln_unbiased_variance": ("const float var = pairwise_sum_f32(v, d, tmp) / df;",
                                "const float var = pairwise_sum_f32(v, d, tmp) / (df - 1.0f);"),
    "adaln_eps_outside_sqrt": ("const float rstd = 1.0f / sqrtf(var + eps);", "const float rstd = 1.0f / (sqrtf(var) + eps);"),
    "adaln_scale_without_one": ("const float a = 1.0f + f32_from_bf16(scale[g * d + i]);",
                                "const float a = f32_from_bf16(scale[g * d + i]);"),
    "adaln_shift_from_scale": ("const float b = f32_from_bf16(shift[g * d + i]);",
                               "const float b = f32_from_bf16(scale[g * d + i]);"),
    "adaln_group_modulo": ("const int64_t g = r / rows_per_group;", "const int64_t g = r % rows_per_group;"),
    "adaln_pairwise_drops_last": ("for (int64_t i = 0; i < p; i++) tmp[i] = (i < n) ? a[i] : 0.0f;",
                                  "for (int64_t i = 0; i < p; i++) tmp[i] = (i < n - 1) ? a[i] : 0.0f;"),
    "adaln_mean_not_subtracted": ("      const float t = v[i] - mu;\n      v[i] = t * t;",
                                  "      const float t = v[i];\n      v[i] = t * t;"),
}

SKIP = {"test_e2m1_exhaustive_core_binades", "test_e2m1_every_fp32_pattern", "test_e8m0_every_positive_finite_value"}


def pin_calls():
    """Every pin of test_oracle_pins as (name, callable taking the oracle module)."""
    calls = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_") or name in SKIP:
            continue
        params = list(inspect.signature(fn).parameters)
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if not marks:
            calls.append((name, (lambda f: lambda orc: f(orc) if "orc" in inspect.signature(f).parameters else f())(fn)))
            continue
        names = [m.args[0] for m in marks]
        for combo in itertools.product(*(m.args[1] for m in marks)):
            kw = dict(zip(names, combo))
            calls.append((f"{name}{list(combo)}", (lambda f, kw: lambda orc: f(orc, **kw))(fn, kw)))
        assert params[0] == "orc"
    return calls


def run_pins(orc):
    failed = []
    for name, call in pin_calls():
        try:
            call(orc)
        except Exception as e:  # an assertion, or an error raised on the planted mistake's output
            failed.append(f"{name}: {type(e).__name__}")
    return failed


def build_copy(orc, tmp_path, text, tag):
    return orc.compile_copy(text, str(tmp_path / f"kq_oracle_{tag}.so"))


def test_unmodified_copy_passes_every_pin(orc, tmp_path):
    text = open(SRC).read()
    with orc.using_library(build_copy(orc, tmp_path, text, "clean")):
        assert run_pins(orc) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(orc, tmp_path, name):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, f"{name}: the text to change must occur exactly once"
    with orc.using_library(build_copy(orc, tmp_path, text.replace(old, new), name)):
        failed = run_pins(orc)
    assert failed, f"no pin caught the planted mistake {name}"
