"""Plants plausible mistakes in copies of the oracle and requires the pins to catch each.

Every mutant below is a one-line edit of oracle/hs2_oracle.cpp (a dropped term, a wrong
sign, index or bound, a swapped operand).  The test compiles the edited copy in a
temporary directory, routes the oracle wrapper to it and runs every pin; at least one
pin must fail.  Nothing here touches a GPU.
"""

import os

import pytest

import oracle
import oracle_pins as P

SRC = os.path.join(os.path.dirname(oracle.__file__), "hs2_oracle.cpp")

MUTANTS = {
    "logit_scale_dropped": ("p[(size_t)h * n + j] = scale * acc;", "p[(size_t)h * n + j] = acc;"),
    "softmax_max_not_subtracted": ("ph[j] = std::exp(ph[j] - m) / l;", "ph[j] = std::exp(ph[j]) / l;"),
    "lse_wrong": ("lse_row[h] = m + std::log(l);", "lse_row[h] = m + l;"),
    "score_not_head_summed": ("s += pj;", "s = pj;"),
    "window_short_by_one": ("for (int64_t j = std::max<int64_t>(0, i - window + 1); j <= i; ++j) sel.push_back(j);",
                            "for (int64_t j = std::max<int64_t>(0, i - window + 2); j <= i; ++j) sel.push_back(j);"),
    "candidates_overlap_window": ("for (int64_t j = 0; j <= i - window; ++j) cand.push_back(j);",
                                  "for (int64_t j = 0; j <= i - window + 1; ++j) cand.push_back(j);"),
    "ties_to_higher_index": ("return a < b;", "return a > b;"),
    "scores_ascending": ("if (score[a] != score[b]) return score[a] > score[b];",
                         "if (score[a] != score[b]) return score[a] < score[b];"),
    "query_position_ignores_offset": ("int64_t i = L - T + t, n = i + 1;", "int64_t i = t + (L > T ? 1 : 0), n = i + 1;"),
    "bridge_operand_transposed": ("acc += xd[k] * bf16_to_f64(w[k]);",
                                  "acc += xd[k] * bf16_to_f64(Wt[((int64_t)k * n_cols + c) % ((int64_t)n_cols * hidden)]);"),
    "fp8_scale_wrong_max": ("double s = amax > 0.0 ? amax / 448.0 : 1.0;", "double s = amax > 0.0 ? amax / 240.0 : 1.0;"),
    "e4m3_bias_wrong": ("(1.0 + m / 8.0) * std::ldexp(1.0, e - 7);", "(1.0 + m / 8.0) * std::ldexp(1.0, e - 8);"),
    "e4m3_ties_to_odd": ("(d == best_d && (c % 2) == 0)", "(d == best_d && (c % 2) == 1)"),
    "bf16_truncates": ("double r = std::nearbyint(x / ulp) * ulp;", "double r = std::trunc(x / ulp) * ulp;"),
    "sparse_uses_v_as_k": ("kd[(size_t)n * D + d] = kv.key(b, sel[n], d);", "kd[(size_t)n * D + d] = kv.val(b, sel[n], d);"),
    "sparse_softmax_not_normalised": ("for (int n = 0; n < ns; ++n) pr[n] = std::exp(pr[n] - m) / l;",
                                      "for (int n = 0; n < ns; ++n) pr[n] = std::exp(pr[n] - m);"),
    "sparse_scale_dropped": ("pr[n] = scale * acc;", "pr[n] = acc;"),
    "sparse_normaliser_drops_last_key": ("for (int n = 0; n < ns; ++n) l += std::exp(pr[n] - m);",
                                         "for (int n = 0; n + 1 < ns; ++n) l += std::exp(pr[n] - m);"),
    "output_uses_next_heads_p": ("for (int d = 0; d < D; ++d) acc[h * D + d] += pj * vj[d];",
                                 "for (int d = 0; d < D; ++d) acc[h * D + d] += p[(size_t)((h + 1) % H) * n + j] * vj[d];"),
    "fp8_value_scale_ignored": ("if (fp8) return e4m3_to_f64(((const uint8_t*)base)[off]) * (double)sc[(int64_t)b * L + j];",
                                "if (fp8) return e4m3_to_f64(((const uint8_t*)base)[off]) * (double)sc[(int64_t)b * L];"),
    "block_score_is_max_not_sum": ("for (int64_t j = 0; j <= last; ++j) bsum[(size_t)(j / block)] += score[j];",
                                   "for (int64_t j = 0; j <= last; ++j) bsum[(size_t)(j / block)] = std::max(bsum[(size_t)(j / block)], score[j]);"),
    "partial_boundary_block_not_counted": ("const int64_t keep = std::min<int64_t>(topk / block, nblk);",
                                           "const int64_t keep = std::min<int64_t>(topk / block, (last + 1) / block);"),
    "block_ties_to_higher_block": ("return b > a;  // equal sums: the lower block first",
                                   "return a > b;  // equal sums: the lower block first"),
    "boundary_block_overlaps_window": ("for (int64_t j = b * block; j < std::min<int64_t>((b + 1) * block, last + 1); ++j)",
                                       "for (int64_t j = b * block; j < (b + 1) * block; ++j)"),
    "slice_sees_one_key_too_many": ("const int64_t n = std::max<int64_t>(0, std::min<int64_t>(L_slice, i + 1));",
                                    "const int64_t n = std::max<int64_t>(0, std::min<int64_t>(L_slice, i + 2));"),
    "slice_score_ignores_given_lse": ("const double ref = lse_in ? lse_in[(size_t)bt * H + h] : lse_row[h];",
                                      "const double ref = lse_row[h];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation site not found exactly once: " + name
    path = tmp_path / "mutant.cpp"
    path.write_text(src.replace(old, new))
    lib = oracle.compile_source(str(path), str(tmp_path / "libmutant.so"))
    caught = []
    with oracle.use_library(lib):
        for check in P.ALL_CHECKS:
            try:
                check()
            except AssertionError:
                caught.append(check.__name__)
    assert caught, "no pin caught mutant " + name
