"""The pins must catch plausible mistakes in the oracle.

Each case copies the oracle's C source, plants one mistake by text
substitution (a dropped term, a wrong sign or index, a transposed layout, a
swapped operand), builds it into a temporary library and runs the whole pin
battery against it: at least one pin must fail.  Nothing here touches a GPU.
"""

import numpy as np
import pytest

import oracle
from tests import oracle_pins

MUTANTS = {
    "gqa_head_mapping": ("const int32_t g = h / group;", "const int32_t g = h % num_kv_heads;"),
    "dropped_scale": ("x[t] = scale * acc;", "x[t] = acc;"),
    "reversed_offset": ("(phys * block_size + t % block_size)",
                        "(phys * block_size + (block_size - 1 - t % block_size))"),
    "head_major_layout": ("((phys * block_size + t % block_size) * num_kv_heads + g)",
                          "((phys * num_kv_heads + g) * block_size + t % block_size)"),
    "no_max_subtraction": ("double w = exp(x[t] - m) / l;", "double w = exp(x[t]) / l * exp(-m);"),
    "no_normalisation": ("double w = exp(x[t] - m) / l;", "double w = exp(x[t] - m);"),
    "sign_error": ("l += exp(x[t] - m);", "l += exp(m - x[t]);"),
    "f16_exponent_bias": ("expo - 25", "expo - 24"),
    "bf16_subnormal_scale": ("ldexp((double)frac, -133)", "ldexp((double)frac, -134)"),
    "cache_write_swapped": ("k_cache[dst] = key[src];", "k_cache[dst] = value[src];"),
    "copy_only_k": ("v_cache[dst * block_elems + e] = v_cache[src * block_elems + e];", ""),
    "context_off_by_one": ("const int32_t ctx = context_lens[s];",
                           "const int32_t ctx = context_lens[s] - 1;"),
    "cache_write_slot_block": ("int64_t offset = slot % block_size;",
                               "int64_t offset = (slot + 1) % block_size;"),
    "table_row_stride": ("block_tables + (int64_t)s * max_blocks_per_seq",
                         "block_tables + (int64_t)s * (max_blocks_per_seq - 1)"),
    "e4m3_exponent_bias": ("ldexp((double)(frac + 8), expo - 10)",
                           "ldexp((double)(frac + 8), expo - 9)"),
    "e4m3_ties_away": ("else pick = (lo & 1) ? hi : lo;", "else pick = hi;"),
    "e4m3_no_saturation": ("if (a >= 448.0) return (uint8_t)(sign | 0x7e);",
                           "if (a >= 448.0) return (uint8_t)(sign | 0x7f);"),
    "fp8_scale_dropped": ("(dec(k_cache[r + d]) * ks)", "(dec(k_cache[r + d]))"),
    "fp8_write_divides_twice": ("const float kq = kx * k_inv;", "const float kq = kx * k_inv * k_inv;"),
    "swap_only_k": ("dst_v[dst * block_bytes + b] = src_v[src * block_bytes + b];", ""),
    "swap_dst_index_of_src": ("dst_k[dst * block_bytes + b] = src_k[src * block_bytes + b];",
                              "dst_k[src % dst_num_blocks * block_bytes + b] = src_k[src * block_bytes + b];"),
    "swap_bad_id_not_flagged": ("            status |= 1;\n            continue;", "            continue;"),
    "fp8_v_scaled_by_k_scale": ("                                       : v_scale;",
                                "                                       : k_scale;"),
    "e4m3_subnormal_scale": ("v = ldexp((double)frac, -9);", "v = ldexp((double)frac, -10);"),
    "e4m3_nan_whole_top_binade": ("if (expo == 15 && frac == 7)", "if (expo == 15)"),
    "f16_subnormal_scale": ("v = ldexp((double)frac, -24);", "v = ldexp((double)frac, -25);"),
    "copy_repeated_dst_not_flagged": ("if (block_mapping[2 * j + 1] == dst && j < i) status |= 8;", ""),
    "copy_dst_read_by_other_not_flagged": (
        "if (block_mapping[2 * j] == dst && block_mapping[2 * j] != block_mapping[2 * j + 1])\n"
        "                status |= 8;", ""),
    "blocked_skips_last_block": ("for (int32_t j = 0; j < nb; ++j) {",
                                 "for (int32_t j = 0; j + 1 < nb; ++j) {"),
    "blocked_block_max_first_token_only": ("t < ctx && t < (j + 1) * block_size",
                                           "t < ctx && t < j * block_size + 1"),
    "int8_unsigned_codes": ("return (double)(int8_t)b;", "return (double)b;"),
    "int8_ties_away": ("else r = fmod(lo, 2.0) == 0.0 ? lo : lo + 1.0;", "else r = lo + 1.0;"),
    "int8_wraps_past_127": ("if (x >= 127.0f) return 127;", "if (x >= 128.0f) return 127;"),
    "int8_nan_saturates": ("if (x != x) return 0;", "if (x != x) return 127;"),
    "int8_decodes_as_e4m3": ("k_scale, v_scale, NULL, NULL, num_threads,\n                           int8_to_f64);",
                             "k_scale, v_scale, NULL, NULL, num_threads,\n                           e4m3_to_f64);"),
    "int8_write_uses_e4m3": ("v_scale, f32_to_int8);", "v_scale, f32_to_e4m3);"),
    # row-scaled one-byte pools
    "rowscale_neighbour_row": ("* block_size + slot % block_size];",
                               "* block_size + (slot + 1) % block_size];"),
    "rowscale_one_scale_for_all_rows": ("row_scale(k_scales, r, num_kv_heads", "row_scale(k_scales, 0, num_kv_heads"),
    "rowscale_token_major_scales": ("((slot / block_size) * num_kv_heads + g) * block_size + slot % block_size]",
                                    "(slot / block_size * block_size + slot % block_size) * num_kv_heads + g]"),
    "rowscale_v_uses_k_scales": ("v_scales ? row_scale(v_scales,", "v_scales ? row_scale(k_scales,"),
    "rowscale_e4m3_top_code_127": ("block_size, num_blocks, dtype, 448.0f, f32_to_e4m3);",
                                   "block_size, num_blocks, dtype, 127.0f, f32_to_e4m3);"),
    "rowscale_stores_amax": ("    *scale = s;\n}", "    *scale = amax;\n}"),
    "rowscale_zero_row_divides_by_zero": ("if (!(s >= FLT_MIN)) {", "if (!(s >= 0.0f)) {"),
    "rowscale_write_scale_index_swapped": ("const int64_t si = (blk * num_kv_heads + g) * block_size + off;",
                                           "const int64_t si = (blk * block_size + off) * num_kv_heads + g;"),
    "rowscale_amax_ignores_sign": ("const float a = fabsf((float)decode(x16[d], dtype));",
                                   "const float a = (float)decode(x16[d], dtype);"),
    "swap_no_conflict_check": ("if (block_mapping[2 * j + 1] == block_mapping[2 * i + 1]) status |= 8;", ""),
}


@pytest.fixture(scope="module")
def source():
    with open(oracle._SRC) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, source, tmp_path):
    old, new = MUTANTS[name]
    assert source.count(old) >= 1, f"mutation site for {name} not found"
    src = tmp_path / "mutant.c"
    src.write_text(source.replace(old, new))
    lib_path = oracle.build(force=True, src=str(src), out=str(tmp_path / "libmutant.so"))
    lib = oracle.load(lib_path)
    caught = []
    with np.errstate(all="ignore"):
        for pin_name, pin in oracle_pins.PINS.items():
            try:
                pin(lib)
            except Exception:            # noqa: BLE001 - any failure counts as caught
                caught.append(pin_name)
    assert caught, f"no pin caught mutant {name}"
