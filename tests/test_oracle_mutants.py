"""Plant plausible mistakes in copies of the oracle and check that some pin catches each.

Each mutant is one textual edit of oracle/gqa_oracle.c (a wrong head->group map, a dropped
scale, an off-by-one length, a missing normalisation, a swapped operand, a wrong sign, a
misplaced append), compiled to a temporary library on the CPU.  The committed oracle is never
modified.
"""
import os

import pytest

import oracle as oracle_mod
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle_mod.__file__), "gqa_oracle.c")

MUTANTS = {
    "group_map_modulo": ("int g = h / r;", "int g = h % H_kv;"),
    "dropped_scale": ("s[t] = scale * acc;", "s[t] = acc;"),
    "skips_appended_row": ("int n = seq_lens[b];\n        if (n < 0 || n > L_max) {",
                           "int n = seq_lens[b] - 1;\n        if (n < 0 || n > L_max) {"),
    "unnormalised": ("double w = s[t] / z;", "double w = s[t];"),
    "weights_keys_not_values": ("out[i] += w * V[(size_t)t * row_stride + i];",
                                "out[i] += w * K[(size_t)t * row_stride + i];"),
    "scores_against_values": ("acc += q[i] * K[(size_t)t * row_stride + i];",
                              "acc += q[i] * V[(size_t)t * row_stride + i];"),
    "wrong_sign": ("s[t] = exp(s[t] - m);", "s[t] = exp(m - s[t]);"),
    "no_max": ("if (s[t] > m) m = s[t];", "(void)0;"),
    "append_off_by_one": ("size_t dst = (((size_t)b * L_max + t) * H_kv + g) * d + i;",
                          "size_t dst = (((size_t)b * L_max + (t ? t - 1 : 0)) * H_kv + g) * d + i;"),
    "append_no_length_update": ("v_cache[dst] = v_new[src];\n            }\n        }\n        seq_lens[b] = t + 1;",
                                "v_cache[dst] = v_new[src];\n            }\n        }\n        seq_lens[b] = t;"),
    "paged_append_no_length_update": ("v_pool[dst + i] = v_new[(size_t)b * row + i];\n        }\n        seq_lens[b] = t + 1;",
                                      "v_pool[dst + i] = v_new[(size_t)b * row + i];\n        }\n        seq_lens[b] = t;"),
    "expand_wrong_head": ("out[((size_t)t * H_q + h) * d + i] = cache_b[((size_t)t * H_kv + g) * d + i];",
                          "out[((size_t)t * H_q + h) * d + i] = cache_b[((size_t)t * H_kv + (H_kv - 1 - g)) * d + i];"),
    "no_divisibility_check": ("H_q % H_kv != 0) return -1;", "0) return -1;"),
    "paged_wrong_offset": ("const double *src = pool + ((size_t)page * page_size + t % page_size) * row;",
                           "const double *src = pool + ((size_t)page * page_size + t / page_size) * row;"),
    "paged_append_wrong_page": ("int page = block_table[(size_t)b * max_pages + t / page_size];\n        if (page < 0 || page >= n_pages) {\n            if (status) *status |= ORACLE_APPEND_OVERFLOW;",
                                "int page = block_table[(size_t)b * max_pages + t % page_size];\n        if (page < 0 || page >= n_pages) {\n            if (status) *status |= ORACLE_APPEND_OVERFLOW;"),
    "multi_not_causal": ("int rows = n - Q + 1 + j;", "int rows = n;"),
    "multi_off_by_one": ("int rows = n - Q + 1 + j;", "int rows = n - Q + j;"),
    "window_off_by_one": ("int first = (window > 0 && n > window) ? n - window : 0;",
                          "int first = (window > 0 && n > window) ? n - window + 1 : 0;"),
    "e4m3_exponent_bias": ("ldexp(1.0 + m / 8.0, e - 7)", "ldexp(1.0 + m / 8.0, e - 8)"),
    "e4m3_subnormal_scale": ("ldexp(m / 8.0, -6)", "ldexp(m / 8.0, -7)"),
    "e4m3_ties_down": ("(dist == best_dist && (c & 1) == 0 && (best & 1) == 1)", "0"),
    "e4m3_no_saturation": ("if (a >= 448.0) return signbit(x) ? 0xFE : 0x7E;",
                           "if (a >= 448.0) return 0x7F;"),
    "quantize_multiplies": ("float quotient = (float)x[at] / scale[g];",
                            "float quotient = (float)x[at] * scale[g];"),
    "dequantize_first_head_scale": ("out[at] = oracle_e4m3_value(codes[at]) * (double)scale[g];",
                                    "out[at] = oracle_e4m3_value(codes[at]) * (double)scale[0];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    lib = oracle_mod.build(str(mutated), str(tmp_path / "libmutant.so"))
    failed = oracle_pins.failing_pins(oracle_mod.Oracle(lib))
    assert failed, f"mutant {name} passed every pin"
