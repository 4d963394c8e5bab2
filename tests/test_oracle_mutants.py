"""Plants plausible mistakes in copies of the oracle and checks that the pins catch each one.

Every mutant is a textual edit of lsa_oracle.c, compiled into a temporary
library and swapped in for the real one while the pin tests run on the CPU.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle
from oracle import build as obuild
from tests import test_oracle_attention as TA
from tests import test_oracle_baselines as TB
from tests import test_oracle_encoder as TE
from tests import test_oracle_label_vote as TL
from tests import test_oracle_select as TS

MUTANTS = {
    "dropped head weight": ("total += bf16_value(w[h]) * dot;", "total += dot;"),
    "dropped ReLU": ("if (dot < 0.0) dot = 0.0;", ""),
    "strict gate": ("if (prob >= 0.5) {", "if (prob > 0.5) {"),
    "sequence offset ignored": ("khat + (size_t)(first + s) * dn", "khat + (size_t)s * dn"),
    "ties to higher index": ("return (x->idx > y->idx) - (x->idx < y->idx);",
                             "return (x->idx < y->idx) - (x->idx > y->idx);"),
    "scale dropped": ("s[j] = scale * dot;", "s[j] = dot;"),
    "window off by one": ("window_start + (j - n_sel)", "window_start + (j - n_sel) + 1"),
    "first window chunk becomes a candidate": ("int first_window_chunk = window_start / LSAO_CHUNK;",
                                               "int first_window_chunk = window_start / LSAO_CHUNK + 1;"),
    "V read with K stride": ("vo[j] = row * (v_pool ? v_row_stride : k_row_stride);", "vo[j] = ko[j];"),
    "nucleus drops crossing element": ("        sel[ord[i].idx] = 1;\n        ++taken;\n        if (cum >= top_p) break;",
                                       "        if (cum >= top_p) break;\n        sel[ord[i].idx] = 1;\n        ++taken;"),
    "union takes only the first indexer": ("for (int i = 0; i < n_idx; ++i) {", "for (int i = 0; i < 1; ++i) {"),
    "union becomes intersection": ("                if (prob >= 0.5)\n                    fetched = 1;",
                                   "                if (prob < 0.5)\n                    fetched = -1;\n"
                                   "                else if (fetched == 0)\n                    fetched = 1;"),
    "random keeps the largest draws": ("neg[c] = -(double)u;", "neg[c] = (double)u;"),
    "random count rounds down": ("((int64_t)n_old * keep_num + keep_den / 2) / keep_den",
                                 "((int64_t)n_old * keep_num) / keep_den"),
    "random draws ignore the sequence": ("((uint64_t)b << 32) + (uint64_t)c", "(uint64_t)c"),
    "encoder W_up transposed": ("w_up[(size_t)o * rank + i]", "w_up[(size_t)i * (Hn * dn) + o]"),
    "encoder head weights from W_down": ("bf16_value(w_head[(size_t)o * d_model + k])",
                                         "bf16_value(w_down[(size_t)o * d_model + k])"),
    "vote threshold strict": ("labels[c] = (uint8_t)(best >= min_layers);", "labels[c] = (uint8_t)(best > min_layers);"),
    "vote counts any step": ("if (count[(size_t)t * n_chunks + c] > best) best = count[(size_t)t * n_chunks + c];",
                             "best += count[(size_t)t * n_chunks + c];"),
}

PINS = [
    lambda o: TS.test_nmi_logit_equals_fused_query_identity(o),
    lambda o: TS.test_nmi_probability_is_library_sigmoid_and_gate_is_logit_sign(o),
    lambda o: TS.test_nmi_structural_plant_is_recovered_exactly(o),
    lambda o: TS.test_nmi_special_cases(o),
    lambda o: TS.test_nmi_sequences_use_their_own_queries(o),
    lambda o: TS.test_nmi_union_keeps_exactly_the_union_of_the_plants(o),
    lambda o: TS.test_nmi_union_each_indexer_alone_keeps_a_different_chunk(o),
    lambda o: TE.test_encoder_equals_library_matrix_products(o),
    lambda o: TE.test_encoder_queries_span_at_most_rank_dimensions(o),
    lambda o: TB.test_recency_only_keeps_no_older_chunk(o),
    lambda o: TB.test_random_selection_is_the_smallest_sequential_splitmix_draws(o),
    lambda o: TB.test_random_count_rounds_half_up_and_respects_the_fraction(o),
    lambda o: TB.test_random_sequences_draw_from_their_own_counters(o),
    lambda o: TS.test_li_score_odd_part_is_linear(o),
    lambda o: TS.test_li_score_special_cases(o),
    lambda o: TS.test_topk_equals_full_library_sort_with_ties(o, 200, 64),
    lambda o: TS.test_topk_all_equal_takes_lowest_indices(o),
    lambda o: TA.test_attention_matches_torch_sdpa(o, 3, 40, 40, 57),
    lambda o: TA.test_decode_step_all_kept_large_k_is_dense_attention(o, False, 5),
    lambda o: TA.test_decode_step_selection_structure(o),
    lambda o: TA.test_decode_step_empty_kept_set_attends_window_only(o),
    lambda o: TL.test_nucleus_uniform_closed_form(o),
    lambda o: TL.test_nucleus_dominant_scores(o),
    lambda o: TL.test_vote_equals_explicit_per_layer_count(o),
    lambda o: TL.test_vote_same_step_versus_any_step(o),
    lambda o: TL.test_vote_threshold_boundary(o),
]


def _compile_mutant(tmp_path, name, old, new):
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, f"mutation site for '{name}' not unique"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-std=c11", "-O1", "-fPIC", "-shared", "-o", str(lib), str(path), "-lm"], check=True)
    return str(lib)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(tmp_path, name):
    old, new = MUTANTS[name]
    libpath = _compile_mutant(tmp_path, name, old, new)
    real = oracle._load()
    mutant = ctypes.CDLL(libpath)
    for fn in ("lsao_nmi_select", "lsao_nmi_select_union", "lsao_select_baseline", "lsao_query_encoder",
               "lsao_li_scores", "lsao_topk_select", "lsao_topk_select_f32",
               "lsao_attention_dense", "lsao_decode_step", "lsao_nucleus", "lsao_label_vote"):
        getattr(mutant, fn).argtypes = getattr(real, fn).argtypes
        getattr(mutant, fn).restype = ctypes.c_int
    caught = []
    oracle._lib = mutant
    try:
        for i, pin in enumerate(PINS):
            try:
                with np.errstate(all="ignore"):
                    pin(oracle)
            except AssertionError:
                caught.append(i)
    finally:
        oracle._lib = real
    assert caught, f"no pin caught the mutant '{name}'"
