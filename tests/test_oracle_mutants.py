"""The pins must reject a broken oracle.

Each case below plants one plausible slip in a copy of the oracle's C source
(a dropped term, a swapped operand, a wrong index or exponent, a wrong
rounding rule), builds it on the CPU, and runs the pin suite against it with
``OPT2S_ORACLE_LIB``.  The suite must fail for every mutant, which shows that
the pins constrain each part of the oracle rather than only re-running it.
"""
import concurrent.futures as cf
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "opt2s_oracle.c")

MUTANTS = {
    "eps_dropped": ("sqrtf(*vi / bc2) + eps", "sqrtf(*vi / bc2)"),
    "eps_inside_sqrt": ("sqrtf(*vi / bc2) + eps", "sqrtf(*vi / bc2 + eps)"),
    "bc1_for_v": ("sqrtf(*vi / bc2)", "sqrtf(*vi / bc1)"),
    "decay_after_update": ("*p = *p * decay - lr * u;", "*p = (*p - lr * u) * decay;"),
    "update_sign": ("*p = *p * decay - lr * u;", "*p = *p * decay + lr * u;"),
    "m2_bias_corrected": ("num = num + alpha * *m2i;", "num = num + alpha * (*m2i / bc1);"),
    "alpha_on_m1": ("num = num + alpha * *m2i;", "num = alpha * num + *m2i;"),
    "one_minus_b3_dropped": ("beta3 * m2 + one_minus_b3 * g", "beta3 * m2 + g"),
    "v_not_squared": ("(one_minus_b2 * g) * g", "(one_minus_b2 * g)"),
    "average_wrong_divisor": ("out[i] = sum / (float)world;",
                              "out[i] = sum / (float)(world + 1);"),
    "average_drops_last_rank": ("for (int q = 1; q < world; q++)",
                                "for (int q = 1; q < world - 1; q++)"),
    "m_uses_beta2": ("*mi = beta1 * m + one_minus_b1 * g;",
                     "*mi = beta2 * m + one_minus_b1 * g;"),
    "bias_exponent_off_by_one": ("pow((double)beta, (double)t)",
                                 "pow((double)beta, (double)(t + 1))"),
    "decay_without_lr": ("1.0 - (double)lr * (double)wd", "1.0 - (double)wd"),
    "m2_aliases_v": ("float *m2 = state1 + n;", "float *m2 = state2;"),
    "skip_zeros_still_decays": (
        "if (skip_zeros && g == 0.0f) continue;",
        "if (skip_zeros && g == 0.0f) { store_param(param, dtype, i, "
        "load_param(param, dtype, i) * decay); continue; }"),
    "ties_away_from_zero": ("if (rem > half || (rem == half && (count & 1))) count++;",
                            "if (rem >= half) count++;"),
    "f16_subnormal_scale": ("ldexp((double)f, -24)", "ldexp((double)f, -25)"),
    "shadow_v_not_squared": ("(1.0 - beta2) * g * g;", "(1.0 - beta2) * g;"),
    "shadow_eps_inside_sqrt": ("sqrt(v[i] / bc2) + eps", "sqrt(v[i] / bc2 + eps)"),
    "shadow_m2_missing_rate": ("beta3 * m2[i] + (1.0 - beta3) * g", "beta3 * m2[i] + g"),
    "unorm_of_grad": ("su += (double)u * (double)u;", "su += (double)g * (double)g;"),
    "pnorm_after_decay": ("sp += (double)p * (double)p;",
                          "sp += (double)(p * decay) * (double)(p * decay);"),
    "unorm_ratio_inverted": ("U > limit ? limit / U : 1.0", "U > limit ? U / limit : 1.0"),
    "unorm_scale_dropped": ("p = p * decay - lr * (scale * u);", "p = p * decay - lr * u;"),
    "unorm_without_sqrt": ("const double U = sqrt(su), P = sqrt(sp);",
                           "const double U = su, P = sp;"),
    "unorm_counts_skipped": (
        "sp += (double)p * (double)p;\n        float g = load_param(grad, dtype, i);\n"
        "        if (skip_zeros && g == 0.0f) continue;\n",
        "sp += (double)p * (double)p;\n        float g = load_param(grad, dtype, i);\n"),
    "lamb_ratio_inverted": ("(float)(P / W)", "(float)(W / P)"),
    "lamb_zero_weight_ratio_zero": ("(P > 0.0 && W > 0.0) ? (float)(P / W) : 1.0f",
                                    "(W > 0.0) ? (float)(P / W) : 1.0f"),
    "lamb_norm_without_decay": ("float w = u + weight_decay * p;\n        sw +=",
                                "float w = u;\n        sw +="),
    "lamb_decay_sign_in_update": ("float w = u + weight_decay * p;\n        p = p - lr",
                                  "float w = u - weight_decay * p;\n        p = p - lr"),
    "lamb_decay_outside_ratio": ("p = p - lr * (ratio * w);",
                                 "p = p - lr * (ratio * u) - lr * (weight_decay * p);"),
    "lamb_ratio_dropped": ("p = p - lr * (ratio * w);", "p = p - lr * w;"),
    "map_bin_edges_not_midpoints": ("(1 << (F + 1)) + 9 * (2 * f + 1)", "(1 << (F + 1)) + 9 * (2 * f)"),
    "map_spare_is_minus_one": ("map[k++] = 1.0f;", "map[k++] = -1.0f;"),
    "map_decades_base_two": ("for (int e = 0; e <= E; e++) D *= 10.0f;",
                             "for (int e = 0; e <= E; e++) D *= 2.0f;"),
    "quantize_ties_upward": ("if (d < bd) { bd = d; best = j; }", "if (d <= bd) { bd = d; best = j; }"),
    "quantize_without_division": ("oracle_quantize(map, x[i] / amax)", "oracle_quantize(map, x[i])"),
    "absmax_kept_from_last_step": ("    *absmax = amax;\n", "    (void)amax;\n"),
    "block_size_1024": ("#define OR_BLOCK8 2048", "#define OR_BLOCK8 1024"),
    "dequant_without_absmax": ("m[k] = smap[q1[i]] * absmax1[b];", "m[k] = smap[q1[i]];"),
    "v_on_signed_map": ("v[k] = umap[q2[i]] * absmax2[b];", "v[k] = smap[q2[i]] * absmax2[b];"),
    "m2_with_m1_absmax": ("smap[q1[n + i]] * absmax1[nblocks + b]", "smap[q1[n + i]] * absmax1[b]"),
    "lamb_counts_skipped": (
        "sp += (double)p * (double)p;\n        float g = load_param(grad, dtype, i);\n"
        "        if (skip_zeros && g == 0.0f) continue;\n        float mi, m2i, vi, u;\n"
        "        element_direction(OR_ADAM",
        "sp += (double)p * (double)p;\n        float g = load_param(grad, dtype, i);\n"
        "        float mi, m2i, vi, u;\n        element_direction(OR_ADAM"),
}


def _build_mutant(name, old, new, tmp):
    import oracle
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    path_c = os.path.join(tmp, f"{name}.c")
    with open(path_c, "w") as f:
        f.write(src.replace(old, new, 1))
    path_so = os.path.join(tmp, f"{name}.so")
    subprocess.run(["gcc", *oracle.CFLAGS, "-o", path_so, path_c, "-lm"],
                   check=True, capture_output=True)
    return path_so


def _run_pins(lib):
    env = dict(os.environ, OPT2S_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q",
                        "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    return r.returncode


def test_every_mutant_is_rejected():
    with tempfile.TemporaryDirectory() as tmp:
        libs = {k: _build_mutant(k, o, n, tmp) for k, (o, n) in MUTANTS.items()}
        with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 2)) as ex:
            codes = dict(zip(libs, ex.map(_run_pins, libs.values())))
    survivors = [k for k, rc in codes.items() if rc == 0]
    assert not survivors, f"pins did not catch: {survivors}"
    assert all(rc == 1 for rc in codes.values()), codes  # failures, not crashes


def test_unmutated_oracle_passes_the_pins():
    import oracle
    assert _run_pins(oracle.build()) == 0
