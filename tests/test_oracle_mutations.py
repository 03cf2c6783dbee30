"""Planted mistakes in a copy of the oracle must each fail at least one pin.

Each mutation below is a plausible slip (a dropped term, a wrong index or
sign, a swapped operand).  The copy is edited and compiled under a temporary
directory; the real oracle source is never touched.
"""
import os

import pytest

import oracle
import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTATIONS = {
    "suffix_keys_dropped": ("if (x >= P) return 1; /* suffix keys: always visible */",
                            "if (x >= P) return 0;"),
    "gqa_modulo_mapping": ("const int kv = h / G;", "const int kv = h % Hkv;"),
    "scale_missing": ("const double scale = 1.0 / sqrt((double)D);", "const double scale = 1.0;"),
    "valid_len_off_by_one": ("if (x >= vl) return 0; /* bucket padding */",
                             "if (x > vl) return 0;"),
    "mask_inverted": ("if (mask_row != NULL && mask_row[x] == 0) return 0;",
                      "if (mask_row != NULL && mask_row[x] != 0) return 0;"),
    "lse_without_max": ("double lse = m + log(z);", "double lse = log(z);"),
    "weights_unnormalised": ("double w = exp(logit_buf[x - key_lo] - lse);",
                             "double w = exp(logit_buf[x - key_lo] - m);"),
    "k_used_as_v": ("const uint16_t *v_row = (x < P) ? vp + (size_t)x * D",
                    "const uint16_t *v_row = (x < P) ? kp + (size_t)x * D"),
    "merge_weight_sign": ("double w = exp(l - total);", "double w = exp(total - l);"),
    "dot_drops_last_term": ("for (int d = 0; d < D; ++d)\n            dot +=",
                            "for (int d = 0; d < D - 1; ++d)\n            dot +="),
    "lse_in_log2": ("double lse = m + log(z);", "double lse = m + log2(z);"),
    "query_head_modulo_kv_heads": ("const int h = (int)((row / S) % Hq);",
                                   "const int h = (int)((row / S) % Hkv);"),
    "normaliser_without_max": ("z += exp(logit_buf[x - key_lo] - m);", "z += exp(logit_buf[x - key_lo]);"),
    "scale_one_over_d": ("const double scale = 1.0 / sqrt((double)D);", "const double scale = 1.0 / (double)D;"),
    "merge_total_is_max": ("double total = m + log(z);", "double total = m;"),
    "merge_skips_first_part": ("for (int s = 0; s < n_parts; ++s) {\n            double l = lse_parts[(size_t)s * rows + r];\n            if (l == -INFINITY) continue;",
                               "for (int s = 1; s < n_parts; ++s) {\n            double l = lse_parts[(size_t)s * rows + r];\n            if (l == -INFINITY) continue;"),
    # prefix-prefill attention under the prefix-causal mask
    "prefill_sees_one_key_too_few": ("const int n = i + 1;", "const int n = i;"),
    "prefill_sees_future_keys": ("const int n = i + 1;", "const int n = vl;"),
    "prefill_computes_padding_rows": ("if (i >= vl) continue; /* padding query: not computed */",
                                      "if (i > vl) continue;"),
    "prefill_gqa_modulo": ("const size_t kv_off = ((size_t)b * Hkv + h / G)",
                           "const size_t kv_off = ((size_t)b * Hkv + h % Hkv)"),
    "prefill_scale_missing": ("logit[j] = inv_sqrt_d * dot;", "logit[j] = dot;"),
    "prefill_lse_without_max": ("const double l = m + log(z);", "const double l = log(z);"),
    "prefill_k_used_as_v": ("const uint16_t *v_row = v + kv_off + (size_t)j * D;",
                            "const uint16_t *v_row = k + kv_off + (size_t)j * D;"),
    # suffix prologue: QKV projection + QK-Norm + RoPE
    "prologue_rope_sign": ("dst[d] = a * c - e * s;", "dst[d] = a * c + e * s;"),
    "prologue_rope_interleaved_pairs": ("const double a = feat[d], e = feat[d + half];",
                                        "const double a = feat[(2 * d) % D], e = feat[(2 * d + 1) % D];"),
    "prologue_rope_angle_exponent": ("pow(theta, -2.0 * (double)d / (double)D)", "pow(theta, -1.0 * (double)d / (double)D)"),
    "prologue_norm_without_mean": ("const double inv_rms = 1.0 / sqrt(ms / (double)D + eps);",
                                   "const double inv_rms = 1.0 / sqrt(ms + eps);"),
    "prologue_key_uses_query_weight": ("const uint16_t *nw = is_q ? qw : kw;", "const uint16_t *nw = qw;"),
    "prologue_values_scaled_by_key_weight": ("for (int d = 0; d < D; ++d) dst[d] = feat[d];\n                    continue;",
                                             "for (int d = 0; d < D; ++d) dst[d] = feat[d] * bf16_bits_to_double(kw[d]);\n                    continue;"),
    "prologue_weight_row_of_next_head": ("const uint16_t *w_row = w + ((size_t)hd * D + d) * (size_t)H;",
                                         "const uint16_t *w_row = w + ((size_t)((hd + 1) % n_heads) * D + d) * (size_t)H;"),
    # post-attention block
    "post_residual_dropped": ("h1[o] = bf16_bits_to_double(h[(size_t)t * Hd + o]) + acc;", "h1[o] = acc;"),
    "post_scale_without_one": ("* (1.0 + bf16_bits_to_double(scale[(size_t)b * Hd + o])) +",
                               "* (bf16_bits_to_double(scale[(size_t)b * Hd + o])) +"),
    "post_shift_dropped": ("+\n                           bf16_bits_to_double(shift[(size_t)b * Hd + o]);",
                           "+\n                           0.0 * bf16_bits_to_double(shift[(size_t)b * Hd + o]);"),
    "post_gelu_cube_dropped": ("(z + 0.044715 * z * z * z)", "(z)"),
    "post_gate_ignored": ("out[(size_t)t * Hd + o] = h1[o] + bf16_bits_to_double(gate[(size_t)b * Hd + o]) * acc;",
                          "out[(size_t)t * Hd + o] = h1[o] + acc;"),
    "post_up_rows_are_gate_rows": ("up += bf16_bits_to_double(wgu[((size_t)F + f) * Hd + c]) * u[c];",
                                   "up += bf16_bits_to_double(wgu[(size_t)f * Hd + c]) * u[c];"),
    "post_norm_without_mean": ("const double inv_rms = 1.0 / sqrt(ms / (double)Hd + eps);",
                               "const double inv_rms = 1.0 / sqrt(ms + eps);"),
    "post_heads_token_major": ("av[hh * D + d] = bf16_bits_to_double(attn[(((size_t)b * Hq + hh) * S + i) * D + d]);",
                               "av[hh * D + d] = bf16_bits_to_double(attn[(((size_t)b * S + i) * Hq + hh) * D + d]);"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(tmp_path, name):
    before, after = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation anchor for {name} not found exactly once"
    mutant_src = tmp_path / "oracle_mutant.c"
    mutant_src.write_text(src.replace(before, after))
    lib = oracle.build(force=True, src=str(mutant_src), out=str(tmp_path / "libmutant.so"))
    mutant = oracle.Oracle(lib)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {name}"
