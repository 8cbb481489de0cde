"""Planted mistakes in the oracle must be caught by its pins (no GPU).

Each case below alters one line of a copy of oracle/ebl_oracle.c the way a
plausible slip would (a flipped sign, a dropped term, a swapped coefficient, a
transposed operand, a reversed tie-break, ...), compiles the copy, and runs the
pins against it: at least one pin has to fail.  The oracle itself is never
modified.  Every planted mistake keeps the copy's memory accesses in bounds,
because the copies run inside the test process.
"""
import os

import pytest

import oracle
from tests import oracle_pins

MUTANTS = {
    "sigmoid_sign": ("return 1.0 / (1.0 + exp(-x));", "return 1.0 / (1.0 + exp(x));"),
    "bias_on_logit": (
        "s[i] = sigmoid_f64(x[i]);\n                key[i] = s[i] + (double)bias[i];",
        "s[i] = sigmoid_f64(x[i] + (double)bias[i]);\n                key[i] = s[i];"),
    "gates_from_keys": ("for (int k = 0; k < K; ++k) gates[t * K + k] = s[sel[k]] / sum;",
                        "for (int k = 0; k < K; ++k) gates[t * K + k] = key[sel[k]] / sum;"),
    "gates_not_normalised": ("gates[t * K + k] = s[sel[k]] / sum;", "gates[t * K + k] = s[sel[k]];"),
    "tie_highest_index": ("if (best < 0 || key[i] > key[best]) best = i; /* equal keys",
                          "if (best < 0 || key[i] >= key[best]) best = i; /* equal keys"),
    "tie_highest_index_f32": ("            if (best < 0 || key[i] > key[best]) best = i;\n        }\n"
                              "        taken[best] = 1;\n        out[k] = best;\n    }\n}\n\n/*\n * Router step, GEMM",
                              "            if (best < 0 || key[i] >= key[best]) best = i;\n        }\n"
                              "        taken[best] = 1;\n        out[k] = best;\n    }\n}\n\n/*\n * Router step, GEMM"),
    "transposed_W": ("x[i] = dot_bf16(h, W + (int64_t)i * d, 1, d);",
                     "x[i] = dot_bf16(h, W + i, Nr, d);"),
    "zloss_transposed_W": ("const double xi = dot_bf16(h, W + (int64_t)i * d, 1, d);",
                           "const double xi = dot_bf16(h, W + i, Nr, d);"),
    "logits_mode_f32_sigmoid": ("s[i] = (float)sigmoid_f64((double)x[i]);",
                                "s[i] = 1.0f / (1.0f + expf(-x[i]));"),
    "smebu_no_recentre": ("double d = db[i] - mean;", "double d = db[i];"),
    "smebu_beta_swapped": ("double m = beta * (double)momentum[i] + (1.0 - beta) * d;",
                           "double m = (1.0 - beta) * (double)momentum[i] + beta * d;"),
    "smebu_no_momentum_decay": ("double m = beta * (double)momentum[i] + (1.0 - beta) * d;",
                                "double m = (double)momentum[i] + (1.0 - beta) * d;"),
    "smebu_v_sign": ("double v = (nbar - (double)counts[i]) / nbar;",
                     "double v = ((double)counts[i] - nbar) / nbar;"),
    "smebu_no_kappa": ("double vt = tanh(kappa * v);", "double vt = tanh(v);"),
    "smebu_v_over_total": ("double v = (nbar - (double)counts[i]) / nbar;",
                           "double v = (nbar - (double)counts[i]) / (double)total;"),
    "smebu_bias_not_added": ("double b = (double)bias[i] + m;\n        momentum[i] = (float)m;\n        bias[i] = (float)b;\n    }\n    free(db);\n    return ORC_OK;\n}\n\n/*\n * Linear",
                             "double b = (double)bias[i] + d;\n        momentum[i] = (float)m;\n        bias[i] = (float)b;\n    }\n    free(db);\n    return ORC_OK;\n}\n\n/*\n * Linear"),
    "sign_recentre_old_b": ("for (int i = 0; i < Nr; ++i) sum += bp[i];",
                            "for (int i = 0; i < Nr; ++i) sum += (double)bias[i];"),
    "sign_of_zero": ("double sgn = (diff > 0.0) ? 1.0", "double sgn = (diff >= 0.0) ? 1.0"),
    "zloss_not_squared": ("total += lse * lse;", "total += lse;"),
    "zloss_no_max_shift": ("const double lse = mx + log(sum);", "const double lse = log(sum);"),
    "maxvio_inverted": ("return (double)mx / (double)mn;", "return (double)mn / (double)mx;"),
    "dispatch_unstable": ("    for (int64_t p = 0; p < P; ++p) {\n        int e = idx[p];",
                          "    for (int64_t p = P - 1; p >= 0; --p) {\n        int e = idx[p];"),
    "dispatch_perm_pair": ("perm[j] = (int32_t)(p / K);", "perm[j] = (int32_t)(p % T);"),
    "tile_counts_first_slot": ("tile_counts[(p / K / tile_tokens) * Nr + idx[p]] += 1;",
                               "tile_counts[(p / K / tile_tokens) * Nr + idx[p - p % K]] += 1;"),
    "gap_sign": ("gap_out[t] = (K == Nr) ? INFINITY : key[sel[K - 1]] - best_rest;",
                 "gap_out[t] = (K == Nr) ? INFINITY : best_rest - key[sel[K - 1]];"),
    "gap_from_first_slot": ("gap_out[t] = (K == Nr) ? INFINITY : key[sel[K - 1]] - best_rest;",
                            "gap_out[t] = (K == Nr) ? INFINITY : key[sel[0]] - best_rest;"),
    "seqbal_unnormalised": ("for (int i = 0; i < Nr; ++i) P[i] += s[i] / row;",
                            "for (int i = 0; i < Nr; ++i) P[i] += s[i];"),
    "seqbal_no_nr_factor": ("f[i] *= (double)Nr / ((double)K * (double)S);",
                            "f[i] *= 1.0 / ((double)K * (double)S);"),
    "seqbal_no_k": ("f[i] *= (double)Nr / ((double)K * (double)S);", "f[i] *= (double)Nr / (double)S;"),
    "seqbal_p_not_averaged": ("            P[i] /= (double)S;\n", ""),
    "seqbal_sum_not_mean": ("    free(P);\n    *loss = total / (double)B;", "    free(P);\n    *loss = total;"),
    "seqbal_gates_as_s_prime": ("for (int j = 0; j < Nr; ++j) row += s[j];",
                                "for (int j = 0; j < K; ++j) row += s[idx[t * K + j]];"),
    "tile_psum_unnormalised": ("psum[(t / tile) * Nr + i] += s[i] / row;", "psum[(t / tile) * Nr + i] += s[i];"),
    "seqbal_tiles_first_sequence": ("for (int64_t j = b * per; j < (b + 1) * per; ++j) {",
                                    "for (int64_t j = 0; j < per; ++j) {"),
    "combine_drops_slot": ("            for (int k = 0; k < K; ++k) {\n                const int64_t row",
                           "            for (int k = 0; k < K - 1; ++k) {\n                const int64_t row"),
}


@pytest.fixture(scope="module")
def src():
    return oracle.source_text()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, src, tmp_path):
    old, new = MUTANTS[name]
    assert src.count(old) == 1, "mutation anchor must match exactly once: %s" % name
    path = oracle.compile_variant(src.replace(old, new), os.path.join(str(tmp_path), "mut_%s.so" % name))
    caught = []
    with oracle.use_library(path):
        for pin in oracle_pins.ALL_PINS:
            try:
                pin()
            except Exception as e:  # AssertionError, or an error the mutant returns
                caught.append((pin.__name__, type(e).__name__))
                break
    assert caught, "planted mistake %r passed every pin" % name
