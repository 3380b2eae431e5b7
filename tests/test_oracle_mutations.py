"""Plant a mistake in a copy of the oracle and check that the pins catch it.

Each mutation is a plausible slip (a dropped term, a wrong sign, a wrong
index, a transposed operand, an off-by-one in a mask).  The copy is compiled
in a temporary directory; the oracle itself is never modified.
"""
import os
import shutil
import subprocess

import pytest

from oracle_pins import ALL_PINS

MUTATIONS = {
    "score_scale_dropped": ("double sij = p->softmax_scale * dot(qi, kj, p->headdim);",
                            "double sij = dot(qi, kj, p->headdim);"),
    "rows_bias_dropped": ("const double sij = score(p, qi, kj, h, i, j);",
                          "const double sij = p->softmax_scale * dot(qi, kj, d);"),
    "causal_off_by_one": ("if (p->causal && j > ii) return 0;", "if (p->causal && j >= ii) return 0;"),
    "window_left_sign": ("j < ii - p->window_left", "j < ii + p->window_left"),
    "window_right_ignored": ("if (p->window_right >= 0 && j > ii + p->window_right) return 0;", ""),
    "alignment_top_left": ("int64_t ii = i + (p->seqlen_k - p->seqlen_q);", "int64_t ii = i;"),
    "gqa_mapping_modulo": ("return h / (p->nheads / p->nheads_kv);", "return h % p->nheads_kv;"),
    "lse_without_max": ("*lse_out = m + log(l);", "*lse_out = log(l);"),
    "softmax_not_normalised": ("exp(s - m) / l;", "exp(s - m);"),
    "alibi_abs_dropped": ("fabs((double)(i + p->seqlen_k - p->seqlen_q - j))",
                          "((double)(i + p->seqlen_k - p->seqlen_q - j))"),
    "alibi_alignment_top_left": ("fabs((double)(i + p->seqlen_k - p->seqlen_q - j))",
                                 "fabs((double)(i - j))"),
    "alibi_wrong_head": ("p->alibi_slopes[h]", "p->alibi_slopes[0]"),
    "merge_weight_not_normalised": ("const double w = exp(lse_parts[s * lrows + lr] - total);",
                                    "const double w = exp(lse_parts[s * lrows + lr] - m);"),
    "merge_lse_without_max": ("const double total = m + log(z);", "const double total = log(z);"),
    "ds_sign_flipped": ("(dp[j] - rowsum)", "(rowsum - dp[j])"),
    "ds_rowsum_dropped": ("(dp[j] - rowsum)", "(dp[j])"),
    "dk_scale_dropped": ("dkj[c] += p->softmax_scale * ds * qi[c];", "dkj[c] += ds * qi[c];"),
    "dv_operand_swapped": ("dvj[c] += pr[j] * zr[j] * doi[c];", "dvj[c] += pr[j] * zr[j] * qi[c];"),
    "dropout_scale_dropped": ("return 256.0 / (256.0 - (double)p->dropout_threshold);",
                              "return 1.0;"),
    "dropout_dv_unmasked": ("dvj[c] += pr[j] * zr[j] * doi[c];", "dvj[c] += pr[j] * doi[c];"),
    "dropout_dp_unmasked": ("? zr[j] * dot(doi, krow(p, v, b, j, g), d)",
                            "? dot(doi, krow(p, v, b, j, g), d)"),
    "dropout_threshold_inclusive": ("if (u < (uint32_t)p->dropout_threshold) return 0.0;",
                                    "if (u <= (uint32_t)p->dropout_threshold) return 0.0;"),
    "dropout_byte_from_row": ("(out[i & 3] >> (8 * (j & 3)))", "(out[j & 3] >> (8 * (i & 3)))"),
    "dropout_head_ignored": ("(uint32_t)((p->batch_base + b) * p->nheads + h)",
                             "(uint32_t)(p->batch_base + b)"),
    "philox_key_not_advanced": ("    k0 += w0;\n", ""),
    "philox_words_swapped": ("    x1 = (uint32_t)p1;\n    x3 = (uint32_t)p0;",
                             "    x1 = (uint32_t)p0;\n    x3 = (uint32_t)p1;"),
    "philox_nine_rounds": ("for (int r = 0; r < 10; ++r)", "for (int r = 0; r < 9; ++r)"),
    "e4m3_bias_off_by_one": ("ldexp(1.0 + m / 8.0, e - 7)", "ldexp(1.0 + m / 8.0, e - 8)"),
    "e4m3_subnormal_scale": ("ldexp(m / 8.0, -6)", "ldexp(m / 8.0, -7)"),
    "e4m3_ties_to_odd": ("(err == best_err && (c & 1) == 0)", "(err == best_err && (c & 1) == 1)"),
    "dq_uses_values": ("dqi[c] += p->softmax_scale * ds * kj[c];",
                       "dqi[c] += p->softmax_scale * ds * krow(p, v, b, j, g)[c];"),
    "scores_wrong_head": ("const double *qi = qrow(p, q, b, i, h);\n  double mx",
                          "const double *qi = qrow(p, q, b, i, 0);\n  double mx"),
}


@pytest.fixture(scope="module")
def oracle_src(oracle_mod):
    with open(os.path.join(os.path.dirname(oracle_mod.__file__), "attn_oracle.c")) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(oracle_mod, oracle_src, tmp_path, name):
    old, new = MUTATIONS[name]
    assert old in oracle_src, f"mutation {name} no longer matches the oracle source"
    src = oracle_src.replace(old, new)
    c = tmp_path / "mutant.c"
    so = tmp_path / "mutant.so"
    c.write_text(src)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                    "-o", str(so), str(c), "-lm"], check=True)
    mutant = oracle_mod.Oracle(str(so))
    caught = []
    for pin in ALL_PINS:
        try:
            pin(mutant)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught mutation {name}"
