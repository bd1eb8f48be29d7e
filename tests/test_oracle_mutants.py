"""Mistakes planted in a copy of the oracle must each be caught by at least one pin.

Each mutant is the oracle's C source with one plausible mistake substituted everywhere its
anchor occurs (a dropped term,
a wrong sign or index, a transposed operand, an off-by-one mask), compiled on the CPU into a
temporary library. The shipped oracle is never modified.
"""
import os

import pytest

import oracle
from oracle import build as obuild
from oracle_checks import ALL_CHECKS

MUTANTS = {
    "rope_sign": ("out[2 * i + 1] = bf16_value(oracle_round_bf16(x0 * s + x1 * c));",
                  "out[2 * i + 1] = bf16_value(oracle_round_bf16(x1 * c - x0 * s));"),
    "rope_theta_exponent": ("pow(base, -2.0 * (double)i / (double)D)", "pow(base, -1.0 * (double)i / (double)D)"),
    "rope_half_split_pairing": ("double x0 = bf16_value(x[2 * i]), x1 = bf16_value(x[2 * i + 1]);",
                                "double x0 = bf16_value(x[i]), x1 = bf16_value(x[i + D / 2]);"),
    "rope_position_offset": ("double angle = (double)pos * theta;", "double angle = (double)(pos + 1) * theta;"),
    "causal_off_by_one": ("if (causal && j > i) visible = 0;", "if (causal && j >= i + 1 + (i > 3)) visible = 0;"),
    "window_off_by_one": ("(long)j < i - window + 1", "(long)j < i - window"),
    "scale_dropped": ("s_row[j] = acc * scale;", "s_row[j] = acc;"),
    "lse_drops_max": ("*lse = m + log(l);", "*lse = log(l);"),
    "values_are_keys": ("const double* vj = vv + (size_t)j * D;", "const double* vj = kk + (size_t)j * D;"),
    "gqa_interleaved_heads": ("if (rb != b || rh / G != g) continue;", "if (rb != b || rh % Hkv != g) continue;"),
    "round_truncates": ("double r = nearbyint(ldexp(ax, -qexp));", "double r = floor(ldexp(ax, -qexp));"),
    "decode_slot_index": ("(size_t)(t % page_size)) * D;", "(size_t)((t + 1) % page_size)) * D;"),
    "decode_query_position": ("attend_row(qq, kk, vv, len, D, (long)len - 1, 1, 0, scale, 0.0, s_row,",
                              "attend_row(qq, kk, vv, len, D, (long)len - 2, 1, 0, scale, 0.0, s_row,"),
    "bwd_no_row_correction": ("const double ds = p * (dp[j] - dsum);", "const double ds = p * dp[j];"),
    "bwd_dk_unscaled": ("my_dk[(size_t)j * D + d] += scale * ds * qq[d];", "my_dk[(size_t)j * D + d] += ds * qq[d];"),
    "bwd_dq_not_rotated_back": ("rope_row_f64(dqr, D, i, rope_base, 1, 0, dq + row * D);",
                                "rope_row_f64(dqr, D, i, rope_base, 0, 0, dq + row * D);"),
    "step_query_position": ("long pos = (long)len - T + t;", "long pos = (long)len - T + t - (t > 0);"),
    "step_append_slot": ("long pos = (long)seq_lens[s] - T + t;", "long pos = (long)seq_lens[s] - T + t + (t == 0);"),
    "step_query_unrotated": ("rope_row(q + row * D, D, pos, rope_base, qq);", "rope_row(q + row * D, D, 0, rope_base, qq);"),
    "alibi_sign": ("s_row[j] -= alibi_slope * (double)(i - j);", "s_row[j] += alibi_slope * (double)(i - j);"),
    "half_split_partner": ("const int a1 = half_split ? i + D / 2 : 2 * i + 1;",
                           "const int a1 = half_split ? D - 1 - i : 2 * i + 1;"),
    "pi_multiplies": ("const double angle = ((double)pos / pos_scale) * theta;",
                      "const double angle = ((double)pos * pos_scale) * theta;"),
    "ntk_exponent": ("pow(ntk_factor, (double)D / (double)(D - 2))", "pow(ntk_factor, 1.0)"),
    "e4m3_bias": ("v = ldexp(1.0 + (double)m / 8.0, e - 7);", "v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "e4m3_subnormal": ("v = ldexp((double)m, -9);", "v = ldexp((double)m, -10);"),
    "normaliser_missing": ("for (int d = 0; d < D; ++d) o[d] /= l;", "for (int d = 0; d < D; ++d) o[d] /= (l + 1e-3);"),
    "bwd_dv_uses_ds": ("my_dv[(size_t)j * D + d] += p * dO[d];", "my_dv[(size_t)j * D + d] += ds * dO[d];"),
    "bwd_dp_uses_keys": ("dp[j] += dO[d] * vv[(size_t)j * D + d];", "dp[j] += dO[d] * kk[(size_t)j * D + d];"),
    "bwd_p_unnormalised": ("for (int j = 0; j < N; ++j) s_row[j] /= lsum;", "for (int j = 0; j < N; ++j) s_row[j] /= 1.0;"),
    "bwd_dk_not_rotated_back": ("rope_row_f64(dk_rot + (size_t)j * D, D, j, rope_base, 1, 0,",
                                "rope_row_f64(dk_rot + (size_t)j * D, D, j, rope_base, 0, 0,"),
    "bwd_row_term_unweighted": ("dsum += s_row[j] * dp[j];", "dsum += dp[j];"),
    "bwd_gqa_interleaved_heads": ("const int h = g * G + r / N, i = r % N;", "const int h = g + (r / N) * Hkv, i = r % N;"),
    "decode_block_table_skipped": ("int32_t pg = block_table[(size_t)s * max_blocks + t / page_size];",
                                   "int32_t pg = (int32_t)((t / page_size) % num_pages);"),
    "decode_cache_layout_head_major": ("(((size_t)pg * Hkv + g) * page_size", "(((size_t)g * num_pages + pg) * page_size"),
    "decode_gqa_interleaved_heads": ("int h = g * G + hh;", "int h = hh * Hkv + g;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(obuild.SRC).read()
    # the same mistake is planted wherever the expression occurs (forward and backward helpers)
    assert src.count(old) >= 1, "mutation anchor not found: %r" % old
    mutant_src = tmp_path / ("oracle_%s.c" % name)
    mutant_src.write_text(src.replace(old, new))
    lib_path = str(tmp_path / ("liboracle_%s.so" % name))
    obuild.build(force=True, src=str(mutant_src), out=lib_path)
    lib = oracle._lib(lib_path)
    caught = []
    for check in ALL_CHECKS:
        try:
            check(lib)
        except Exception as e:  # an AssertionError or an oracle error status
            caught.append((check.__name__, type(e).__name__))
    assert caught, "mutant %s passed every pin" % name
