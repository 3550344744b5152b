"""The oracle's pins must catch plausible slips.

Each case plants one mistake in a copy of the oracle's C source (on the CPU,
in a temporary directory), builds it, and runs the pin suite against the
broken copy: the suite has to fail.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

MUTANTS = {
    "ties_to_higher_index": ("if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;",
                             "if (!taken[e] && (best < 0 || l[e] >= l[best])) best = e;"),
    "selects_smallest": ("if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;",
                         "if (!taken[e] && (best < 0 || l[e] < l[best])) best = e;"),
    "silu_on_w3_branch": ("h[f] = silu(a) * b;", "h[f] = a * silu(b);"),
    "dropped_w3_term": ("h[f] = silu(a) * b;", "h[f] = silu(a);"),
    "w2_transposed": ("acc += bf16_bits_to_double(r2[f]) * h[f];",
                      "acc += bf16_bits_to_double(W2[(size_t)f * d + o]) * h[f];"),
    "softmax_sign": ("        w[j] = exp(l[sel[j]] - m);\n        s += w[j];\n    }\n    for (int j = 0; j < k; ++j) w[j] /= s;\n}",
                     "        w[j] = exp(m - l[sel[j]]);\n        s += w[j];\n    }\n    for (int j = 0; j < k; ++j) w[j] /= s;\n}"),
    "bias_ignored": ("if (bias) acc += bias[e];", "if (bias) acc += 0.0 * bias[e];"),
    "shared_expert_dropped": ("for (int i = 0; i < d; ++i) o[i] += y[i];",
                              "for (int i = 0; i < d; ++i) o[i] += 0.0 * y[i];"),
    "unnormalised_weights": ("for (int j = 0; j < k; ++j) w[j] /= s;\n}",
                             "for (int j = 0; j < k; ++j) w[j] /= 1.0;\n}"),
    "gap_from_top1": ("*gap = l[sel[k - 1]] - l[next];", "*gap = l[sel[0]] - l[next];"),
    "gap_next_is_smallest": ("if (!taken[e] && (next < 0 || l[e] > l[next])) next = e;",
                             "if (!taken[e] && (next < 0 || l[e] < l[next])) next = e;"),
    "gap_skips_a_place": ("*gap = l[sel[k - 1]] - l[next];",
                          "*gap = (k > 1 ? l[sel[k - 2]] : l[sel[k - 1]]) - l[next];"),
    "softmax_all_normalised_over_selected": (
        "for (int e = 0; e < E; ++e) s += exp(l[e] - m);",
        "for (int e = 0; e < k; ++e) s += exp(l[sel[e]] - m);"),
    "sigmoid_weight_sign": ("for (int j = 0; j < k; ++j) w[j] = sigmoid(l[sel[j]]);",
                            "for (int j = 0; j < k; ++j) w[j] = sigmoid(-l[sel[j]]);"),
    "sigmoid_gate_uses_silu": ("if (act_mode == 1) h[f] = sigmoid(a) * b;",
                               "if (act_mode == 1) h[f] = silu(a) * b;"),
    "sigmoid_gate_on_w3": ("if (act_mode == 1) h[f] = sigmoid(a) * b;",
                           "if (act_mode == 1) h[f] = a * sigmoid(b);"),
    "capacity_off_by_one": ("keep[(size_t)t * k + j] = cnt[e] < cap;",
                            "keep[(size_t)t * k + j] = cnt[e] <= cap;"),
    "capacity_reverse_token_order": ("            for (int t = 0; t < T; ++t)\n                for (int j = 0; j < k; ++j) {\n                    int e = sel_all",
                                     "            for (int t = T - 1; t >= 0; --t)\n                for (int j = 0; j < k; ++j) {\n                    int e = sel_all"),
    "e4m3_exponent_bias": ("ldexp(8.0 + m, e - 10)", "ldexp(8.0 + m, e - 11)"),
    "e4m3_subnormal_scale": ("ldexp((double)m, -9)", "ldexp((double)m, -10)"),
    "fp8_scale_of_wrong_row": ("for (int i = 0; i < d; ++i) b += s3[f] * e4m3_to_double(r3[i]) * xt[i];",
                               "for (int i = 0; i < d; ++i) b += s3[0] * e4m3_to_double(r3[i]) * xt[i];"),
    "fp8_w2_scale_by_hidden_index": ("acc += s2[o] * e4m3_to_double(r2[f]) * h[f];",
                                     "acc += s2[f % d] * e4m3_to_double(r2[f]) * h[f];"),
    "ep_tokens_reversed": ("for (int t = 0; t < T_of[r]; ++t)\n                    for (int j = 0; j < k; ++j) {",
                           "for (int t = T_of[r] - 1; t >= 0; --t)\n                    for (int j = 0; j < k; ++j) {"),
    "ep_slot_major": ("for (int t = 0; t < T_of[r]; ++t)\n                    for (int j = 0; j < k; ++j) {",
                      "for (int j = 0; j < k; ++j)\n                    for (int t = 0; t < T_of[r]; ++t) {"),
    "ep_offsets_shifted": ("seg[e - q * El + 1] = row;", "seg[e - q * El] = row;"),
    "ep_rows_continue_across_owners": ("int32_t row = 0;\n        int32_t *seg",
                                       "static int32_t row = 0;\n        int32_t *seg"),
    "entropy_threshold_flipped": ("*k_used = H > ENTROPY_THRESHOLD ? k : k - 1;",
                                  "*k_used = H > ENTROPY_THRESHOLD ? k - 1 : k;"),
    "entropy_without_temperature": ("#define ENTROPY_TAU 0.1", "#define ENTROPY_TAU 1.0"),
    "entropy_weights_unnormalised": ("for (int j = 0; j < k; ++j) w[j] = exp((l[sel[j]] - m) / ENTROPY_TAU) / s;",
                                     "for (int j = 0; j < k; ++j) w[j] = exp((l[sel[j]] - m) / ENTROPY_TAU);"),
    "entropy_in_bits": ("if (pe > 0.0) H -= pe * log(pe);", "if (pe > 0.0) H -= pe * log2(pe);"),
    "logits_without_bias": ("if (logits) memcpy(logits + (size_t)t * E, l, sizeof(double) * (size_t)E);",
                            "if (logits) { memcpy(logits + (size_t)t * E, l, sizeof(double) * (size_t)E);"
                            " if (bias) for (int e = 0; e < E; ++e) logits[(size_t)t * E + e] -= bias[e]; }"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = src.replace(old, new, 1)
    c = tmp_path / "mutant.c"
    so = tmp_path / "libmutant.so"
    c.write_text(mutated)
    subprocess.run(["gcc", "-O1", "-std=c11", "-fopenmp", "-shared", "-fPIC", "-o", str(so),
                    str(c), "-lm"], check=True)
    env = dict(os.environ, MOE_ORACLE_LIB=str(so), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"planted mistake '{name}' passed every pin:\n{r.stdout[-2000:]}"
