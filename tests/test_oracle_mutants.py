"""Plant plausible mistakes in copies of the oracle and require that the pins
catch every one (CPU only). Each mutant is the oracle's C source with one
textual replacement, compiled to a temporary library."""
import os

import pytest

import oracle
import oracle_pins

MUTANTS = {
    "high_nibble_read_as_low": ("q[64 * g + 32 + l] = Q[32 * g + l] >> 4;",
                                "q[64 * g + 32 + l] = Q[32 * g + l] & 15;"),
    "nibble_halves_swapped": ("q[64 * g + l] = Q[32 * g + l] & 15;",
                              "q[64 * g + l] = Q[32 * g + l] >> 4;"),
    "group_stride_32": ("q[64 * g + l] = Q[32 * g + l] & 15;",
                        "q[32 * g + l] = Q[32 * g + l] & 15;"),
    "scale_top_bits_wrong_byte": ("((S[j - 4] >> 6) << 4)", "((S[j - 3] >> 6) << 4)"),
    "min_low_bits_wrong_nibble": ("mn[j] = (S[j + 4] >> 4)", "mn[j] = (S[j + 4] & 15)"),
    "scale_mask_5_bits": ("sc[j] = S[j] & 63;", "sc[j] = S[j] & 31;"),
    "min_sign_flipped": ("out[t] = dsc * (float)q[t] - dm;", "out[t] = dsc * (float)q[t] + dm;"),
    "min_term_dropped": ("out[t] = dsc * (float)q[t] - dm;", "out[t] = dsc * (float)q[t];"),
    "subblock_of_64": ("int j = t / 32;", "int j = t / 64;"),
    "dmin_used_for_scale": ("float dsc = d * (float)sc[j];", "float dsc = dmin * (float)sc[j];"),
    "half_bias_off_by_one": ("expo - 25", "expo - 24"),
    "half_subnormal_scale": ("ldexp((double)frac, -24)", "ldexp((double)frac, -25)"),
    "d_dmin_fields_swapped": ("*d_bits = u16le(sb + 0);", "*d_bits = u16le(sb + 2);"),
    "x_block_stride_dropped": ("x + (int64_t)i * k + b * QK", "x + (int64_t)i * k"),
    "abs_sum_signed": ("sa += fabs(p);", "sa += p;"),
    "embed_token_off_by_one": ("if (token >= rows)", "if (token > rows)"),
    "embed_size_check_relaxed": ("if (table_bytes != expected ||", "if (table_bytes < expected ||"),
    "embed_width_rule_dropped": ("if (hidden == 0 || hidden % QK != 0)", "if (hidden == 0)"),
    "embed_shape_rule_dropped": ("if (cols != hidden)\n        return Q4K_ORACLE_EMBED_SHAPE;", ""),
    "embed_scale_not_applied": ("(float)((double)wv[t] * (double)embed_scale)", "wv[t]"),
    "embed_wrong_row_stride": ("table + (token * nsb + b) * SB_BYTES", "table + (token + b) * SB_BYTES"),
    "half_ties_to_odd": ("pick = (lo & 1) ? lo + 1 : lo;", "pick = (lo & 1) ? lo : lo + 1;"),
    "half_ties_away": ("pick = (lo & 1) ? lo + 1 : lo;", "pick = lo + 1;"),
    "half_truncates": ("    else if (dhi < dlo)\n        pick = lo + 1;\n", ""),
    "half_overflow_early": ("if (v >= 65520.0)", "if (v >= 65504.0)"),
    "half_nan_to_inf": ("return (uint16_t)(sign | 0x7E00);", "return (uint16_t)(sign | 0x7C00);"),
    "mirror_row_stride_dropped": ("out[r * k + b * QK + t] = q4k_oracle_float_to_half(v[t]);",
                                  "out[b * QK + t] = q4k_oracle_float_to_half(v[t]);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    with open(oracle.SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    path = os.path.join(tmp_path, "mutant.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    mutant = oracle.Oracle(oracle.build(path, os.path.join(tmp_path, "libmutant.so"), force=True))
    caught = []
    # The golden file is the oracle's own output, so it does not count as a catch.
    for check in [c for c in oracle_pins.ALL_CHECKS if c is not oracle_pins.check_golden]:
        try:
            check(mutant)
        except AssertionError:
            caught.append(check.__name__)
    assert caught, f"no pin catches the planted mistake {name}"
