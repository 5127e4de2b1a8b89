"""Planted mistakes in copies of the oracle must each fail at least one pin.

Each mutant is the oracle's C source with one plausible error written in
(a dropped scale, an off-by-one or reversed mask, the wrong value columns, a
wrong page or head index, a dropped max or the wrong base in lse, unnormalised
weights, a sign slip or a dropped part in the merge).  The copy is
compiled on the CPU into a temporary directory; the real oracle is untouched.
"""
import os

import pytest

import oracle
from oracle_pins import ALL_PINS

MUTANTS = {
    "no_scale": ("s[j - first] = softmax_scale * acc;", "s[j - first] = acc;"),
    "mask_off_by_one": ("int last = causal ? L - s_q + i : L - 1;",
                        "int last = causal ? L - s_q + i - 1 : L - 1;"),
    "value_from_rope_end": ("orow[c] += w * bf16_to_double(vrow[c]);",
                            "orow[c] += w * bf16_to_double(vrow[c + (d - dv)]);"),
    "page_index": ("block_table[(size_t)b * max_pages + j / page_size]",
                   "block_table[(size_t)b * max_pages + 0 * (j / page_size)]"),
    "slot_index": ("(size_t)(j % page_size)", "(size_t)((j + 1) % page_size)"),
    "kv_head": ("const int g = h / heads_per_kv;", "const int g = h % h_kv;"),
    "lse_drops_max": ("*lse_out = m + log(z);", "*lse_out = log(z);"),
    "merge_sign": ("const double w = exp(part_lse[k] - total);",
                   "const double w = exp(total - part_lse[k]);"),
    "rope_dims_dropped": ("for (int c = 0; c < d; ++c) acc +=", "for (int c = 0; c < dv; ++c) acc +="),
    "append_position": ("const long long pos = (long long)L + t;", "const long long pos = (long long)L + t + 1;"),
    "append_slot": ("(size_t)(pos % page_size)", "(size_t)((pos + 63) % page_size)"),
    "unabsorbed_wv_transposed": ("t += wv[(size_t)r * dc + k] * c[k];", "t += wv[(size_t)k * dvo + r] * c[k];"),
    "unabsorbed_rope_dropped": ("for (int r = 0; r < dr; ++r) acc += qr[r] * c[dc + r];",
                                "for (int r = 0; r < dr; ++r) acc += 0.0 * qr[r] * c[dc + r];"),
    "causal_query_reversed": ("int last = causal ? L - s_q + i : L - 1;",
                              "int last = causal ? L - 1 - i : L - 1;"),
    "non_causal_drops_last": ("int last = causal ? L - s_q + i : L - 1;",
                              "int last = causal ? L - s_q + i : L - 2;"),
    "lse_base_2": ("*lse_out = m + log(z);", "*lse_out = m + log2(z);"),
    "weights_unnormalised": ("const double w = exp(s[j - first] - m) / z;",
                             "const double w = exp(s[j - first] - m);"),
    "empty_row_lse_zero": ("*lse_out = -INFINITY;\n      continue;", "*lse_out = 0.0;\n      continue;"),
    "value_head_zero": ("const uint16_t* vrow = kv_row(kv, block_table, max_pages, b, j, g, h_kv, d, page_size);",
                        "const uint16_t* vrow = kv_row(kv, block_table, max_pages, b, j, 0, h_kv, d, page_size);"),
    "window_end_off_by_one": ("if (key_hi && key_hi[b] - 1 < last) last = key_hi[b] - 1;",
                              "if (key_hi && key_hi[b] - 1 < last) last = key_hi[b];"),
    "merge_skips_first_part": ("for (int k = 0; k < n; ++k) {\n    const double w = exp(part_lse[k] - total);",
                               "for (int k = 1; k < n; ++k) {\n    const double w = exp(part_lse[k] - total);"),
    "append_head": ("uint16_t* dst =\n            kvcache + (((size_t)page * page_size + (size_t)(pos % page_size)) * h_kv + g)",
                    "uint16_t* dst =\n            kvcache + (((size_t)page * page_size + (size_t)(pos % page_size)) * h_kv + 0)"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(oracle.SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    path = os.path.join(tmp_path, f"mut_{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = oracle.OracleLib(oracle.build(force=True, src=path, out=os.path.join(tmp_path, f"{name}.so")))
    failures = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError) as e:
            failures.append(pin.__name__)
    assert failures, f"mutant {name} passed every pin"
