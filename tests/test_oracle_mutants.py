"""Plant plausible mistakes in copies of the oracle and check the pins catch them.

Each mutant is a one-line textual change to ``oracle/hsa_oracle.c`` (a dropped
term, a wrong sign or index, swapped operands, a wrong tie-break...).  The
mutant is compiled to a temporary library and ``tests/test_oracle.py`` is run
against it in a child process; the run must fail.  The mistakes are planted in
the CPU oracle only.
"""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "hsa_oracle.c")

MUTANTS = {
    "group_sum_not_mean": ("qbar[j] = acc / (double)G;", "qbar[j] = acc;"),
    "group_uses_first_head": ("for (int h = 0; h < G; ++h) acc += q_row",
                              "for (int h = 0; h < 1; ++h) acc += q_row"),
    "no_scale_in_chunk_logits": ("logit[r] = scale * dot(q, k + r * d, d);",
                                 "logit[r] = dot(q, k + r * d, d);"),
    "own_chunk_excludes_self": ("t - first + 1, d,", "t - first, d,"),
    "own_chunk_dropped": ("if (own_chunk) {", "if (0) {"),
    "own_chunk_visible": ("const int64_t nvis = c; ", "const int64_t nvis = c + (c < Nc); "),
    "tie_break_highest_index": ("if (a->index < b->index) return -1;",
                                "if (a->index < b->index) return 1;"),
    "ascending_scores": ("if (a->score > b->score) return -1;",
                         "if (a->score > b->score) return 1;"),
    "fusion_not_normalised": ("softmax_inplace(wk, (int)nsel);", ";"),
    "softmax_wrong_sign": ("logit[r] = exp(logit[r] - m);", "logit[r] = exp(m - logit[r]);"),
    "k_v_swapped": ("chunk_attention(q_h, k_bg + first * d, v_bg + first * d, S, d, scale,",
                    "chunk_attention(q_h, v_bg + first * d, k_bg + first * d, S, d, scale,"),
    "landmark_mean_without_sqrtS": ("l[j] = sqrt((double)S) * mean;", "l[j] = mean;"),
    "chunk_offset_off_by_one": ("const int64_t first = sel[kk] * S;\n",
                                "const int64_t first = sel[kk] * S + (sel[kk] > 0 ? -1 : 1);\n"),
    "fusion_weight_from_group_query": ("wk[kk] = scale * dot(q_h, lm_bg", "wk[kk] = scale * dot(qbar, lm_bg"),
    "decode_weights_unnormalised": ("softmax_inplace(wk, nsel);", ";"),
    # near-tie gap: the next pair down the ranking (off by one)
    "gap_off_by_one": ("gap_val = nvis > topk ? cand[topk - 1].score - cand[topk].score : INFINITY;",
                       "gap_val = nvis > topk + 1 ? cand[topk].score - cand[topk + 1].score : INFINITY;"),
    "decode_gap_off_by_one": ("gap[bg] = Nc > topk ? cand[topk - 1].score - cand[topk].score : INFINITY;",
                              "gap[bg] = Nc > topk + 1 ? cand[topk].score - cand[topk + 1].score : INFINITY;"),
    # near-tie scale: the magnitude of a score's terms taken as |score|
    "score_magnitude_without_abs": ("for (int j = 0; j < n; ++j) acc += fabs(x[j] * y[j]);",
                                    "for (int j = 0; j < n; ++j) acc += x[j] * y[j];"),
    # retrieval variants: each token decides for itself instead of its block start
    "variant_block_start_ignored": ("const int64_t t0 = (t / interval) * interval;",
                                    "const int64_t t0 = t;"),
    # retrieval variants: the union softmax leaves out the own chunk, or its last key
    "variant_union_drops_own_chunk": ("if (own_chunk)\n                        for (int64_t jj = own_first; jj <= t; ++jj)",
                                      "if (0)\n                        for (int64_t jj = own_first; jj <= t; ++jj)"),
    "variant_union_own_excludes_self": ("for (int64_t jj = own_first; jj <= t; ++jj) keyrow[nk++] = jj;",
                                        "for (int64_t jj = own_first; jj < t; ++jj) keyrow[nk++] = jj;"),
    # retrieval variants: mean pooling over the block's first token only
    "variant_mean_pool_first_only": ("const int64_t u1 = pool_mean ? t1 : t0 + 1;",
                                     "const int64_t u1 = t0 + 1;"),
    # variable-length chunks: own chunk starting at a multiple of S, landmark without sqrt(|C|)
    "varlen_own_chunk_fixed_start": ("const int64_t own_first = bounds ? bounds[c] : c * S;",
                                     "const int64_t own_first = c * S;"),
    "varlen_landmark_without_sqrt": ("lm_dhsa[(bg * Nc + i) * d + j] = sqrt((double)n) * (sum / (double)n);",
                                     "lm_dhsa[(bg * Nc + i) * d + j] = sum / (double)n;"),
    # forced selection: chunks not visible from the row are kept
    "forced_visibility_filter_dropped": ("if (f[kk] >= 0 && f[kk] < nvis) sel[nsel++] = f[kk];",
                                         "if (f[kk] >= 0 && f[kk] < Nc) sel[nsel++] = f[kk];"),
    # forced selection: slots taken in reverse order
    "forced_slots_reversed": ("const int32_t *f = forced_idx + (r * Hkv + g) * topk;",
                              "int32_t f[64]; for (int kk = 0; kk < topk; ++kk) f[kk] = forced_idx[(r * Hkv + g) * topk + topk - 1 - kk];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    msrc = tmp_path / "mutant.c"
    msrc.write_text(src.replace(old, new))
    lib = oracle.build(str(msrc), str(tmp_path / "libmutant.so"))
    env = dict(os.environ, HSA_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"no pin caught mutant {name}:\n{r.stdout[-2000:]}"
