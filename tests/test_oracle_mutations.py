"""The pins must reject a plausibly wrong oracle.

Each case plants one mistake in a copy of the oracle's C source (on the CPU),
builds it, and runs the pin suite against that build; the suite must fail.
"""
import os
import subprocess
import sys

import pytest

import oracle.zq_oracle as zo

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = {
    "round_down": ("return nearbyintf(v);", "return floorf(v);"),
    "ties_away": ("return nearbyintf(v);", "return roundf(v);"),
    "scale_qmax_plus_one": ("return amax / (float)qmax;", "return amax / (float)(qmax + 1);"),
    "group_ceil": ("return (int)(((int64_t)o * g) / N);", "return (int)(((int64_t)o * g + N - 1) / N);"),
    "nibble_swap": ("packed[(size_t)o * (K / 2) + 4 * m + i] = (uint8_t)(lo | (hi << 4));",
                    "packed[(size_t)o * (K / 2) + 4 * m + i] = (uint8_t)(hi | (lo << 4));"),
    "ln_mean_sign": ("float d = h2f(x[k]) - mean;", "float d = h2f(x[k]) + mean;"),
    "ln_var_drop_mean": ("float d = h2f(x[k0]) - mean;", "float d = h2f(x[k0]);"),
    "ln_unbiased_var": ("float var = chunk_tree_sum(x, K, 1, mean) / (float)K;",
                        "float var = chunk_tree_sum(x, K, 1, mean) / (float)(K - 1);"),
    "ln_one_pass_var": ("float var = chunk_tree_sum(x, K, 1, mean) / (float)K;",
                        "float var = chunk_tree_sum(x, K, 1, 0.0f) / (float)K - mean * mean;"),
    "ln_tree_skips_pad": ("for (int c = 0; c < n; c += 2 * step) v[c] = v[c] + v[c + step];",
                          "for (int c = 0; c + step < n - 1; c += 2 * step) v[c] = v[c] + v[c + step];"),
    "gemm_reversed_k": ("for (int k = 0; k < K; ++k) s += (int64_t)a[k] * (int64_t)b[k];",
                        "for (int k = 0; k < K; ++k) s += (int64_t)a[k] * (int64_t)b[K - 1 - k];"),
    "dequant_row_scale_swapped": ("v = v * s_grp[zqo_group_of(o, N, g)];\n            v = v + (bias ? h2f(bias[o]) : 0.0f);\n            Y[(size_t)t * N + o] = f2h(v);\n        }\n    return 0;\n}\n\n/* GEMM + dequant",
                                  "v = v * s_grp[zqo_group_of(N - 1 - o, N, g)];\n            v = v + (bias ? h2f(bias[o]) : 0.0f);\n            Y[(size_t)t * N + o] = f2h(v);\n        }\n    return 0;\n}\n\n/* GEMM + dequant"),
    "dequant_bias_reversed": ("v = v + (bias ? h2f(bias[o]) : 0.0f);\n            Y[(size_t)t * N + o] = f2h(v);\n        }\n    return 0;\n}\n\n/* GEMM",
                              "v = v + (bias ? h2f(bias[N - 1 - o]) : 0.0f);\n            Y[(size_t)t * N + o] = f2h(v);\n        }\n    return 0;\n}\n\n/* GEMM"),
    "token_clamp_126": ("s_tok[t] = eq2_scale(amax, 127, &inv);\n        for (int k = 0; k < K; ++k) q[(size_t)t * K + k] = (int8_t)eq2_quantize(h2f(y[k]), inv, 127);",
                        "s_tok[t] = eq2_scale(amax, 127, &inv);\n        for (int k = 0; k < K; ++k) q[(size_t)t * K + k] = (int8_t)eq2_quantize(h2f(y[k]), inv, 126);"),
    "gelu_sqrt2_inverted": ("erfc(-v / sqrt(2.0))", "erfc(-v * sqrt(2.0))"),
    "gelu_no_half": ("return 0.5 * v * erfc", "return v * erfc"),
    "gelu_sign_flipped": ("erfc(-v / sqrt(2.0))", "erfc(v / sqrt(2.0))"),
    "act_bias_ignored": ("if (bias) v = v + h2f(bias[k]);", "if (bias) v = v + 0.0f * h2f(bias[k]);"),
    "static_ema_swapped": ("xmax = momentum * xmax + (1.0f - momentum) * bmax;",
                           "xmax = (1.0f - momentum) * xmax + momentum * bmax;"),
    "static_range_max_only": ("*A = fmaxf(fabsf(xmax), fabsf(xmin));", "*A = fabsf(xmax);"),
    "act_gelu_skipped": ("act == 1 ? d2h(zqo_gelu((double)v)) : f2h(v)", "act == 1 ? f2h(v) : f2h(v)"),
    "a16_weights_transposed": ("(double)q[(size_t)o * K + k];", "(double)q[(size_t)k * N + o];"),
    "a16_bias_dropped": ("(bias ? (double)h2f(bias[o]) : 0.0);", "0.0;"),
    "a16_group_by_token": ("sum * (double)s_grp[zqo_group_of(o, N, g)]", "sum * (double)s_grp[zqo_group_of(t % N, N, g)]"),
}


@pytest.fixture(scope="module")
def mutant_runs(tmp_path_factory):
    src = open(zo._SRC).read()
    d = tmp_path_factory.mktemp("mutants")
    procs = {}
    for name, (old, new) in MUTATIONS.items():
        assert src.count(old) == 1, name
        c = d / f"{name}.c"
        c.write_text(src.replace(old, new))
        so = d / f"{name}.so"
        subprocess.check_call(["gcc", *zo.CFLAGS, str(c), "-o", str(so), "-lm"])
        env = dict(os.environ, ZQ_ORACLE_LIB=str(so))
        procs[name] = subprocess.Popen(
            [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
             os.path.join(ROOT, "tests", "test_oracle_pins.py")],
            cwd=ROOT, env=env, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)
    return {name: (p.wait(timeout=600), p.stdout.read().decode()) for name, p in procs.items()}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_reject_mutant(mutant_runs, name):
    rc, out = mutant_runs[name]
    assert rc == 1, f"mutant {name} was not caught (rc={rc}):\n{out[-2000:]}"
