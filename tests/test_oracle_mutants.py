"""Every plausible slip in the oracle must fail at least one pin.

Each case copies the oracle's C source, plants one mistake (a dropped term, a
wrong sign, index or operand), compiles the copy and runs the pins of
tests/oracle_pins.py against it.  A mutant that passes every pin would mean the
pins cannot tell that mistake from the real oracle.
"""

import pytest

import oracle
import oracle_pins

MUTANTS = {
    "rms_sum_not_mean": ("sqrt(ss / (double)d + eps)", "sqrt(ss + eps)"),
    "rms_eps_outside_sqrt": ("sqrt(ss / (double)d + eps)", "sqrt(ss / (double)d) + eps"),
    "rms_gamma_reversed": ("h3o_bf16_to_double(gamma[i])", "h3o_bf16_to_double(gamma[d - 1 - i])"),
    "rope_sign": ("row[i0] = x0 * c - x1 * s;", "row[i0] = x0 * c + x1 * s;"),
    "rope_freq_width": ("-2.0 * (double)i / (double)width[axis]", "-2.0 * (double)i / (double)d"),
    "rope_section_offset": ("int start[3] = {0, sec_t, sec_t + sec_h};", "int start[3] = {0, sec_h, sec_t + sec_h};"),
    "rope_axis_swap": ("(double)p[axis] * f", "(double)p[2 - axis] * f"),
    "rope_1d_freq": ("pow(theta, -2.0 * (double)i / (double)d);\n            rotate_pair(row, 2 * i",
                     "pow(theta, -1.0 * (double)i / (double)d);\n            rotate_pair(row, 2 * i"),
    "rope_pair_stride": ("rotate_pair(row, 2 * i, (double)p[0] * f);", "rotate_pair(row, i, (double)p[0] * f);"),
    "attn_scale_dropped": ("sc[j - j0] = scale * dot;", "sc[j - j0] = dot;"),
    "attn_q_dot_v": ("dot += qd[i] * kd[j * d + i];", "dot += qd[i] * vd[j * d + i];"),
    "attn_lse_no_max": ("lse[r * n_heads + h] = mx + log(den);", "lse[r * n_heads + h] = log(den);"),
    "attn_no_max_shift": ("double p = exp(sc[j - j0] - mx);", "double p = exp(sc[j - j0]);"),
    "attn_boundary": ("t < cu_seqlens[s + 1])) ++s;", "t <= cu_seqlens[s + 1])) ++s;"),
    "attn_no_normalise": ("out[i] = acc[i] / den;", "out[i] = acc[i];"),
    "kv_scale_dropped": ("s_row[j - kb] = scale * qk;", "s_row[j - kb] = qk;"),
    "kv_lse_no_max": ("lse[t * n_heads + h] = m + log(z);", "lse[t * n_heads + h] = log(z);"),
    "kv_segment_keys": ("const int64_t kb = cu_k[seg], ke = cu_k[seg + 1];",
                        "const int64_t kb = cu_q[seg], ke = cu_q[seg + 1];"),
    "merge_weight_unnormalised": ("const double w = exp(lse_parts[p * n_rows + r] - L);",
                                  "const double w = exp(lse_parts[p * n_rows + r] - mx);"),
    "merge_lse_is_max": ("const double L = mx + log(den);", "const double L = mx;"),
    "qkv_weight_transposed": ("acc += xin[c] * h3o_bf16_to_double(w[f * dim_in + c]);",
                              "acc += xin[c] * h3o_bf16_to_double(w[c * dim_in + f % dim_in]);"),
    "qkv_bias_dropped": ("feat[i] = bias ? acc + h3o_bf16_to_double(bias[f]) : acc;", "feat[i] = acc;"),
    "qkv_k_uses_gamma_q": ("part == 1 ? gamma_k : NULL;", "part == 1 ? gamma_q : NULL;"),
    "qkv_part_offset": ("const int64_t f = part * hd + (int64_t)h * d + i;",
                        "const int64_t f = part * hd + (int64_t)h * d + (i ^ 1);"),
    "bs_query_block_size": ("const int64_t list = ((int64_t)b * n_heads + h) * n_qb + t / block_q;",
                            "const int64_t list = ((int64_t)b * n_heads + h) * n_qb + t / block_k;"),
    "bs_list_order": ("const int64_t list = ((int64_t)b * n_heads + h) * n_qb + t / block_q;",
                      "const int64_t list = ((int64_t)h * batch + b) * n_qb + t / block_q;"),
    "bs_key_block_off_by_one": ("if (!seen[j / block_k]) continue;\n                const int64_t kr",
                                "if (!seen[(j + 1) / block_k]) continue;\n                const int64_t kr"),
    "bs_key_batch_order": ("const int64_t kr = ((b * n_kv + j) * n_heads + h) * (int64_t)d;",
                           "const int64_t kr = ((j * batch + b) * n_heads + h) * (int64_t)d;"),
    "bs_lse_no_max": ("lse[r * n_heads + h] = m + log(z);", "lse[r * n_heads + h] = log(z);"),
    "bs_scale_dropped": ("s_row[j] = scale * qk;", "s_row[j] = qk;"),
    "bf16_round_half_up": ("nearbyint(ax / quantum)", "floor(ax / quantum + 0.5)"),
    "bf16_subnormal_quantum": ("quantum = ldexp(1.0, -133);", "quantum = ldexp(1.0, -134);"),
    "bf16_mantissa_bits": ("quantum = ldexp(1.0, e - 1 - 7);", "quantum = ldexp(1.0, e - 1 - 8);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(oracle.SOURCE).read()
    assert src.count(old) == 1, "mutation anchor not found exactly once: %r" % old
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = oracle.build(str(path), str(tmp_path / ("lib_%s.so" % name)), force=True)
    orc = oracle.Oracle(lib)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError) as e:
            caught.append(pin.__name__)
    assert caught, "mutant %s passed every pin" % name
