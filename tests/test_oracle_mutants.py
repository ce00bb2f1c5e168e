"""The pins must catch plausible mistakes in the oracle.

Each case plants one mistake in a copy of the oracle's C source (on the CPU,
never in the real oracle), builds it, and runs the pin suite against that
build: the suite has to fail.  Together the cases cover every step of the
oracle: the transform, the quantiser, the GEMM and the dequantisation.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "convrot_oracle.c")
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

MUTANTS = {
    "butterfly_sign": ("v[j + h] = u - w;", "v[j + h] = w - u;"),
    "missing_last_stage": ("for (int h = 1; h < b; h <<= 1) {", "for (int h = 1; h < b / 2; h <<= 1) {"),
    "round_half_away": ("float r = rintf(v);", "float r = roundf(v);"),
    "product_rounded_once": ("float r = rintf(v); /*", "float r = (float)rint((double)z[k] * (double)inv); /*"),
    "scale_over_128": ("*s = amax / 127.0f;", "*s = amax / 128.0f;"),
    "inverse_scale_128": ("float inv = 127.0f / amax;", "float inv = 128.0f / amax;"),
    "zero_row_scale_one": ("        *s = 0.0f;\n        memset(q, 0, (size_t)K);", "        *s = 1.0f;\n        memset(q, 0, (size_t)K);"),
    "bf16_widen": ("uint32_t u = (uint32_t)h << 16;", "uint32_t u = (uint32_t)h << 15;"),
    "gemm_transposed_operand": ("const int8_t *bb = B + n * ldb;", "const int8_t *bb = B + (m % N) * ldb;"),
    "dequant_drops_1_over_b": ("double v = (double)acc[m * N + n] * (double)s_a[m] * (double)s_b[n] * alpha;",
                               "double v = (double)acc[m * N + n] * (double)s_a[m] * (double)s_b[n];"),
    "dequant_drops_bias": ("            if (bias) v += (double)bias[n];\n            if (gelu) v = gelu_f64(v);\n            y[m * N + n] = v;",
                           "            if (gelu) v = gelu_f64(v);\n            y[m * N + n] = v;"),
    "gelu_half_missing": ("return 0.5 * y * erfc(-y / sqrt(2.0));", "return y * erfc(-y / sqrt(2.0));"),
    "gelu_erfc_sign": ("return 0.5 * y * erfc(-y / sqrt(2.0));", "return 0.5 * y * erfc(y / sqrt(2.0));"),
    "silu_sign": ("static double silu_f64(double g) { return g / (1.0 + exp(-g)); }",
                  "static double silu_f64(double g) { return g / (1.0 + exp(g)); }"),
    "swiglu_halves_swapped": ("else if (act == 2) v = silu_f64(v) * (double)bf16_bits_to_f32(h[K + k]);",
                              "else if (act == 2) v = (double)bf16_bits_to_f32(h[K + k]) * 0 + silu_f64((double)bf16_bits_to_f32(h[K + k])) * v;"),
    "regular_output_drops_factor_2": ("v[j] = t - 2.0f * x0;", "v[j] = t - x0;"),
    "regular_missing_last_stage": ("for (int st = 1; st < b; st *= 4) {\n        for (int i = 0; i < b; i += 4 * st) {",
                                   "for (int st = 1; st < b / 4; st *= 4) {\n        for (int i = 0; i < b; i += 4 * st) {"),
    "regular_h4_sign": ("if ((i / st) % 4 == (j / st) % 4) sign = -sign;", "if ((i / st) % 4 != (j / st) % 4) sign = -sign;"),
    "amax_skips_first": ("for (int64_t k = 0; k < K; ++k) {\n        float a = fabsf(z[k]);", "for (int64_t k = 1; k < K; ++k) {\n        float a = fabsf(z[k]);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    from oracle import oracle as O
    subprocess.check_call(["gcc", *O.CFLAGS, "-o", str(lib), str(mutant), "-lm"])
    env = dict(os.environ, CONVROT_ORACLE_LIB=str(lib), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", PINS, "-x", "-q", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"the pins did not notice the planted mistake '{name}':\n{r.stdout[-2000:]}"
