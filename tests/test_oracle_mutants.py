"""The oracle pins must catch plausible mistakes.

Each case plants one mistake in a copy of oracle.c (on the CPU, in a temporary
directory), builds it, and runs the pin suite against that build in a child
process. Every mutant must fail at least one pin; the unmodified source must pass.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

# (name, exact text in oracle.c, replacement, occurrence to replace: 0 = first, 1 = second)
MUTANTS = [
    ("gate_dropped", "g * oracle_bf16_to_double(xr[c])", "oracle_bf16_to_double(xr[c])", 0),
    ("residual_sign", "oracle_bf16_to_double(rr[c]) + g *", "oracle_bf16_to_double(rr[c]) - g *", 0),
    ("norm_on_unrounded_r", "v[c] = oracle_bf16_to_double(rb);", "v[c] = exact;", 0),
    ("double_rounding_r", "oracle_bf16_rne(exact)", "oracle_bf16_rne((double)(float)exact)", 0),
    ("eps_outside_sqrt", "1.0 / sqrt(second + eps)", "1.0 / (sqrt(second) + eps)", 0),
    ("eps_ignored", "1.0 / sqrt(second + eps)", "1.0 / sqrt(second + 1e-5)", 0),
    ("unbiased_variance", "second /= (double)D;", "second /= (double)(D > 1 ? D - 1 : 1);", 1),
    ("mean_off_by_one", "mu /= (double)D;", "mu /= (double)(D + 1);", 0),
    ("rms_uses_abs", "second += v[c] * v[c];", "second += fabs(v[c]);", 0),
    ("scale_shift_swapped", "(1.0 + oracle_bf16_to_double(sr[c])) + oracle_bf16_to_double(tr[c])",
     "(1.0 + oracle_bf16_to_double(tr[c])) + oracle_bf16_to_double(sr[c])", 0),
    ("modulation_without_one", "n * (1.0 + oracle_bf16_to_double(sr[c]))", "n * (oracle_bf16_to_double(sr[c]))", 0),
    ("weight_added", "n = n * oracle_bf16_to_double(weight[c]);", "n = n + oracle_bf16_to_double(weight[c]);", 0),
    ("bias_dropped", "n = n + oracle_bf16_to_double(bias[c]);", "n = n;", 0),
    ("fp32_weight_cast_to_bf16", "if (weight_f32) n = n * (double)weight_f32[c];",
     "if (weight_f32) n = n * oracle_bf16_to_double(oracle_bf16_rne((double)weight_f32[c]));", 0),
    ("frame_index_mod", "l / tokens_per_frame : 0", "l % tokens_per_frame : 0", 0),
    ("ties_away", "(frac == 0.5 && fmod(whole, 2.0) == 1.0)", "(frac == 0.5)", 0),
    ("rounding_truncates", "if (frac > 0.5 || (frac == 0.5 && fmod(whole, 2.0) == 1.0)) whole += 1.0;", "", 0),
    ("subnormal_quantum", "if (qexp < -133) qexp = -133;", "if (qexp < -126) qexp = -126;", 0),
    ("bias_before_weight",
     "        if (weight) n = n * oracle_bf16_to_double(weight[c]);\n"
     "        if (weight_f32) n = n * (double)weight_f32[c];\n"
     "        if (bias) n = n + oracle_bf16_to_double(bias[c]);\n",
     "        if (bias) n = n + oracle_bf16_to_double(bias[c]);\n"
     "        if (weight) n = n * oracle_bf16_to_double(weight[c]);\n"
     "        if (weight_f32) n = n * (double)weight_f32[c];\n", 0),
    ("norm_of_x_not_r", "v[c] = oracle_bf16_to_double(rb);", "v[c] = oracle_bf16_to_double(xr[c]);", 0),
    ("rms_with_layernorm_statistics", "if (is_rms) {", "if (0) {", 0),
    ("double_rounding_y", "yr[c] = oracle_bf16_rne(yv);", "yr[c] = oracle_bf16_rne((double)(float)yv);", 0),
    ("batch_stride_ignored", "return b * st[0] + f * st[1] + l * st[2];", "return f * st[1] + l * st[2];", 0),
    ("gate_on_residual", "oracle_bf16_to_double(rr[c]) + g * oracle_bf16_to_double(xr[c])",
     "g * oracle_bf16_to_double(rr[c]) + oracle_bf16_to_double(xr[c])", 0),
    ("shift_with_scale_strides", "shift + row_offset(shift_st, b, f, l)", "shift + row_offset(scale_st, b, f, l)", 0),
    ("frame_from_flat_row", "l / tokens_per_frame : 0", "row / tokens_per_frame : 0", 0),
    ("layernorm_not_centred", "double n = (v[c] - mu) * rho;", "double n = v[c] * rho;", 0),
    ("eps_as_floor", "1.0 / sqrt(second + eps)", "1.0 / sqrt(second > eps ? second : eps)", 0),
    ("rho_in_float", "double rho = 1.0 / sqrt(second + eps);",
     "double rho = (double)(1.0f / sqrtf((float)(second + eps)));", 0),
    ("mean_accumulated_in_float", "for (int64_t c = 0; c < D; ++c) mu += v[c];",
     "for (int64_t c = 0; c < D; ++c) mu = (double)(float)(mu + v[c]);", 0),
    ("variance_accumulated_in_float", "second += (v[c] - mu) * (v[c] - mu);",
     "second = (double)(float)(second + (v[c] - mu) * (v[c] - mu));", 0),
    # a NaN statistic clamped away (fmax returns the non-NaN operand): NaN rows turn finite
    ("nan_statistic_clamped", "1.0 / sqrt(second + eps)", "1.0 / sqrt(fmax(second, 0.0) + eps)", 0),
]


def _apply(text, old, new, occurrence):
    pos = -1
    for _ in range(occurrence + 1):
        pos = text.index(old, pos + 1)
    return text[:pos] + new + text[pos + len(old):]


def _run_pins(lib_path):
    env = dict(os.environ, ORACLE_LIB=lib_path, OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
           os.path.join(ROOT, "tests", "test_oracle_pins.py")]
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)


def _build(directory, text, name):
    sys.path.insert(0, ROOT)
    from oracle.build import build

    src = os.path.join(directory, f"{name}.c")
    with open(src, "w") as f:
        f.write(text)
    return build(src, os.path.join(directory, f"lib{name}.so"))


@pytest.fixture(scope="module")
def pin_runs(tmp_path_factory):
    """Every mutant (and the unmodified oracle) built and run against the pins, the
    builds and pin runs in parallel (each is its own subprocess)."""
    from concurrent.futures import ThreadPoolExecutor

    directory = str(tmp_path_factory.mktemp("mutants"))
    text = open(SRC).read()
    cases = [("clean", text)] + [(name, _apply(text, old, new, occ)) for name, old, new, occ in MUTANTS]

    def one(case):
        name, src = case
        return name, (src != text or name == "clean"), _run_pins(_build(directory, src, name))

    workers = max(2, min(8, (os.cpu_count() or 2) // 2))
    with ThreadPoolExecutor(workers) as ex:
        return {name: (changed, res) for name, changed, res in ex.map(one, cases)}


def test_unmodified_oracle_passes_pins(pin_runs):
    _, res = pin_runs["clean"]
    assert res.returncode == 0, res.stdout[-2000:]


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_mutant_is_caught(pin_runs, name):
    changed, res = pin_runs[name]
    assert changed, f"mutant {name} did not change the source"
    assert res.returncode != 0, f"mutant {name} passed every pin:\n{res.stdout[-1500:]}"
