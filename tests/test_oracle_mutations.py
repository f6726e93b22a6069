"""The pins must catch plausible mistakes in the oracle.

Each case plants one mistake in a copy of the oracle's C source (on the CPU),
builds it, and runs the pin suite against that copy: the suite must fail.
"""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = {
    "stage_order_descending": ("for (int h = 1; h < ROT_N; h <<= 1) {",
                               "for (int h = ROT_N / 2; h >= 1; h >>= 1) {"),
    "butterfly_sign_swapped": ("v[i + h] = a - c;", "v[i + h] = c - a;"),
    "no_normalisation": ("v[i] = v[i] * 0.0625f;", "v[i] = v[i] * 1.0f;"),
    "reciprocal_instead_of_division": ("float t = y[k] / s;", "float t = y[k] * (1.0f / s);"),
    "round_half_away": ("float r = nearbyintf(t);", "float r = roundf(t);"),
    "truncate": ("float r = nearbyintf(t);", "float r = truncf(t);"),
    "max_without_abs": ("float a = fabsf(y[k]);", "float a = y[k];"),
    "scale_over_qmax_plus_1": ("float s = amax / qmax;", "float s = amax / (qmax + 1.0f);"),
    "gemm_transposed_weight": ("const int8_t *b = Qw + n * K;\n            int32_t s = 0;\n            for (int64_t k = 0; k < K; ++k)\n                s += (int32_t)a[k] * (int32_t)b[k];\n            acc[m * N + n] = s;",
                               "int32_t s = 0;\n            for (int64_t k = 0; k < K; ++k)\n                s += (int32_t)a[k] * (int32_t)Qw[(k % N) * K + (n % K)];\n            acc[m * N + n] = s;"),
    "epilogue_drops_weight_scale": ("    f = f * sw;\n", "    (void)sw;\n"),
    "epilogue_bias_dropped": ("    f = f + b;\n", "    (void)b;\n"),
    "bf16_truncates": ("if (rest > 0x8000u || (rest == 0x8000u && (kept & 1u)))", "if (0)"),
    "bf16_ties_away": ("if (rest > 0x8000u || (rest == 0x8000u && (kept & 1u)))", "if (rest >= 0x8000u)"),
    "gelu_cubic_coefficient": ("(x + 0.044715 * (x * x * x))", "(x + 0.04715 * (x * x * x))"),
    "gelu_drops_factor_two": ("return x / (1.0 + exp(-2.0 * u));", "return x / (1.0 + exp(-u));"),
    "silu_wrong_sign": ("return x / (1.0 + exp(-x));", "return x / (1.0 + exp(x));"),
    "act_tiny_ties_to_even": ("double q = (t - lo == 0.5) ? lo + 1.0 : nearbyint(t);",
                              "double q = nearbyint(t);"),
    "f64_bf16_truncates": ("double q = nearbyint(ldexp(a, -qe));", "double q = floor(ldexp(a, -qe));"),
    "f64_bf16_no_subnormal_spacing": ("if (qe < -133)\n        qe = -133;", "(void)0;"),
    "int4_qmax_8": ("oracle_quant_row_q(buf, K, 7.0f, q, s_w + n);", "oracle_quant_row_q(buf, K, 8.0f, q, s_w + n);"),
    "int4_nibbles_swapped": ("(uint8_t)(((uint8_t)q[2 * j] & 0xFu) | (((uint8_t)q[2 * j + 1] & 0xFu) << 4));",
                             "(uint8_t)(((uint8_t)q[2 * j + 1] & 0xFu) | (((uint8_t)q[2 * j] & 0xFu) << 4));"),
    "int4_unpack_no_sign": ("Q8[2 * i] = (int8_t)(lo >= 8 ? lo - 16 : lo);", "Q8[2 * i] = (int8_t)lo;"),
    "e2m1_ties_away_from_zero": ("if (d < bestd || (d == bestd && (c & 1u) == 0)) {", "if (d <= bestd) {"),
    "e4m3_truncates": ("float k = nearbyintf(v / u);", "float k = floorf(v / u);"),
    "nvfp4_scale_tile_lines_swapped": ("return tile * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4;",
                                       "return tile * 512 + ((r % 128) / 32) * 16 + (r % 32) * 4 + c % 4;"),
    "nvfp4_nibble_order_swapped": ("q[k / 2] = (uint8_t)(q[k / 2] | (code << (4 * (k & 1))));",
                                   "q[k / 2] = (uint8_t)(q[k / 2] | (code << (4 * ((k + 1) & 1))));"),
    "nvfp4_tensor_scale_constant": ("const float s_t = amax / 2688.0f;", "const float s_t = amax / 2682.0f;"),
    "nvfp4_block_amax_signed": ("                        if (fabsf(y[i]) > ab)\n                            ab = fabsf(y[i]);",
                                "                        if (y[i] > ab)\n                            ab = y[i];"),
    "act_not_rounded_to_bf16": ("buf[k] = oracle_bf16_to_f32(oracle_act_bf16(act, row[k]));",
                                "buf[k] = (float)oracle_act_f64(act, oracle_bf16_to_f32(row[k]));"),
    "rmsnorm_eps_outside_sqrt": ("double inv = 1.0 / sqrt(ss / (double)K + (double)eps);",
                                 "double inv = 1.0 / (sqrt(ss / (double)K) + (double)eps);"),
    "rmsnorm_sum_not_mean": ("double inv = 1.0 / sqrt(ss / (double)K + (double)eps);",
                             "double inv = 1.0 / sqrt(ss + (double)eps);"),
    "rmsnorm_drops_a_square": ("    for (int64_t k = 0; k < K; ++k) {\n        double v = (double)oracle_bf16_to_f32(h[k]);\n        double t = v * v;",
                               "    for (int64_t k = 1; k < K; ++k) {\n        double v = (double)oracle_bf16_to_f32(h[k]);\n        double t = v * v;"),
    "rmsnorm_weight_dropped": ("if (g) v = v * (double)oracle_bf16_to_f32(g[k]);", "(void)g;"),
    "rmsnorm_residual_subtracted": ("h[k] = R ? oracle_f32_to_bf16_rne(x + oracle_bf16_to_f32(R[m * ldr + k]))",
                                    "h[k] = R ? oracle_f32_to_bf16_rne(x - oracle_bf16_to_f32(R[m * ldr + k]))"),
    "rmsnorm_no_alt_offered": ("        *alt = o;\n", "        (void)o;\n"),
}


# Which pin file is meant to catch each kind of mistake (the others are not
# run for it, to keep the suite short).
PIN_FILES = {
    "act": ["test_oracle_act_pins.py"],
    "int4": ["test_oracle_w4a4_pins.py"],
    "nvfp4": ["test_oracle_nvfp4_pins.py"],
    "core": ["test_oracle_pins.py"],
    "rmsnorm": ["test_oracle_rmsnorm_pins.py"],
}


def _pins_for(name: str):
    if name.startswith(("gelu", "silu", "act_", "f64_")):
        return PIN_FILES["act"]
    if name.startswith("int4"):
        return PIN_FILES["int4"]
    if name.startswith(("e2m1", "e4m3", "nvfp4")):
        return PIN_FILES["nvfp4"]
    if name.startswith("rmsnorm"):
        return PIN_FILES["rmsnorm"]
    return PIN_FILES["core"]


def _run_mutant(workdir: str, name: str):
    old, new = MUTATIONS[name]
    src = open(oracle._SRC).read()
    if old not in src:
        return name, None, f"mutation {name} no longer applies"
    mut = os.path.join(workdir, f"{name}.c")
    with open(mut, "w") as f:
        f.write(src.replace(old, new, 1))
    so = os.path.join(workdir, f"lib{name}.so")
    subprocess.check_call(["gcc", *oracle.CFLAGS, mut, "-o", so, "-lm"],
                          stderr=subprocess.DEVNULL)
    env = dict(os.environ, CONVROT_ORACLE_LIB=so, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        *[os.path.join(ROOT, "tests", f) for f in _pins_for(name)]],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return name, r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def mutant_runs(tmp_path_factory):
    """Every mutant built and its pins run once, several at a time (each run
    is a separate process that loads that mutant's library)."""
    from concurrent.futures import ThreadPoolExecutor

    workdir = str(tmp_path_factory.mktemp("mutants"))
    workers = max(1, min(8, (os.cpu_count() or 2) // 2))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        results = list(ex.map(lambda n: _run_mutant(workdir, n), sorted(MUTATIONS)))
    return {name: (rc, out) for name, rc, out in results}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(mutant_runs, name):
    rc, out = mutant_runs[name]
    assert rc is not None, out
    assert rc != 0, f"pins did not catch {name}:\n{out}"
