"""The pins must catch plausible mistakes in the oracle.

Each case copies the oracle source to a temporary directory, plants one
mistake by text substitution, builds it with gcc and runs a pin against it
(CPU only).  The pin must fail; the unmodified oracle passes the same pins in
the other test files.
"""
import subprocess

import pytest

import oracle
import test_oracle_cycle as tc
import test_oracle_exact as tex
import test_oracle_filter as tf
import test_oracle_linear as tl
import test_oracle_params as tpa
import test_oracle_philox as tp
import test_oracle_tree as tt

SRC = (oracle._HERE / "uno_ref.c").read_text()

MUTATIONS = {
    "philox multiplier": ("(uint64_t)0xD2511F53u * (uint64_t)c0", "(uint64_t)0xD2511F55u * (uint64_t)c0",
                          lambda: [tp.test_philox_known_answers(*row) for row in tp._kat_rows()]),
    "uniform word order": ("((uint64_t)x[0] << 21) | (uint64_t)(x[1] >> 11)",
                           "((uint64_t)x[1] << 21) | (uint64_t)(x[0] >> 11)",
                           lambda: [tp.test_uniform_counter_layout(*row) for row in tp._kat_rows()]),
    "top-k tie order": ("    return (a->id > b->id) - (a->id < b->id);\n}\n\nstatic int cmp_id_asc",
                        "    return (a->id < b->id) - (a->id > b->id);\n}\n\nstatic int cmp_id_asc",
                        tf.test_greedy_is_argmax_with_lowest_id_on_ties),
    "temperature multiplies": ("w[j] = exp(((double)e[j].v - (double)e[0].v) / T);",
                               "w[j] = exp(((double)e[j].v - (double)e[0].v) * T);",
                               tf.test_full_softmax_when_nothing_is_cut),
    "top-p includes next mass": ("if (!(m < top_p)) break;", "if (!(m + w[j] / S < top_p)) break;",
                                 lambda: tf.test_top_p_is_shortest_prefix_reaching_top_p(1.0, 50, 0.95)),
    "renormalise skipped": ("out[j].v = (float)(w[j] / W);", "out[j].v = (float)(w[j]);",
                            tf.test_compact_output_invariants),
    "accept test inverted": ("accept = (u * a < px);", "accept = (u * px < a);",
                             lambda: tl.test_linear_output_is_the_target_process(4, 2, 1.0, 4, 1.0, 11)),
    "residual sign flipped": ("double d = (double)pi_pr[j] - lookup_prob(qi_ids, qi_pr, qc, pi_ids[j]);",
                              "double d = lookup_prob(qi_ids, qi_pr, qc, pi_ids[j]) - (double)pi_pr[j];",
                              lambda: tl.test_linear_output_is_the_target_process(4, 2, 1.0, 4, 1.0, 11)),
    "residual not clipped": ("qc, pi_ids[j]);\n                wts[j] = d > 0.0 ? d : 0.0;",
                             "qc, pi_ids[j]);\n                wts[j] = d > 0.0 ? d : -d;",
                             lambda: tl.test_linear_output_is_the_target_process(4, 2, 1.0, 4, 1.0, 11)),
    # With full supports (every token in supp q) this mistake changes nothing,
    # so the sampling pin on such rows passes it; the exact enumeration on
    # rows whose supports differ catches it.
    "residual over supp q only": ("qc, pi_ids[j]);\n                wts[j] = d > 0.0 ? d : 0.0;",
                                  "qc, pi_ids[j]);\n                wts[j] = (d > 0.0 && lookup_prob(qi_ids, qi_pr, qc, pi_ids[j]) > 0.0) ? d : 0.0;",
                                  lambda: tex.test_linear_exact_distribution_is_the_target_process(*tex.LINEAR_CASES[1])),
    "bonus from wrong row": ("for (int j = 0; j < p_cnt[B]; ++j) wts[j] = (double)p_probs[(size_t)B * (size_t)cap + (size_t)j];",
                             "for (int j = 0; j < p_cnt[B]; ++j) wts[j] = (double)p_probs[(size_t)(B - 1) * (size_t)cap + (size_t)j];",
                             lambda: tl.test_linear_output_is_the_target_process(4, 2, 1.0, 4, 1.0, 11)),
    "accept and residual share a draw": ("uno_ref_uniform(seed, first_request + (uint32_t)r, (uint32_t)i, DRAW_RESIDUAL, cycle);",
                                         "uno_ref_uniform(seed, first_request + (uint32_t)r, (uint32_t)i, DRAW_ACCEPT, cycle);",
                                         lambda: tl.test_linear_output_is_the_target_process(4, 2, 1.0, 4, 1.0, 11)),
    "tree tie by deeper first": ("if (a->depth != b->depth) return a->depth < b->depth;",
                                 "if (a->depth != b->depth) return a->depth > b->depth;",
                                 tt.test_ties_break_by_depth_then_parent_then_rank),
    "tree children from wrong marginal": ("score[idx] * (double)cand[(size_t)t * (size_t)K + (size_t)j].p",
                                          "score[idx] * (double)cand[(size_t)(t > 0 ? t - 1 : 0) * (size_t)K + (size_t)j].p",
                                          lambda: tt.test_expansion_is_the_top_scoring_paths(3, 3, 20, 2)),
    "tree descends on any child": ("if (pa[cnd] == j && tk[cnd] == y) {", "if (pa[cnd] == j) {",
                                   lambda: tt.test_tree_output_is_the_target_process(4, 2, 2, 5, 1.0, 4, 1.0, 31)),
    "joint mass from the top-k set alone": ("for (int64_t j = kk; j < n; ++j) S += exp(",
                                            "for (int64_t j = n; j < n; ++j) S += exp(",
                                            lambda: [tpa.test_joint_order_worked_example(*c) for c in tpa.WORKED]),
    "joint mass counts the top-k twice": ("for (int64_t j = kk; j < n; ++j) S += exp(",
                                          "for (int64_t j = 0; j < n; ++j) S += exp(",
                                          lambda: tpa.test_geometric_row_closed_form(37, 1.0)),
    "filter params indexed by position": ("int64_t rq = r / rows_per_request;", "int64_t rq = r % rows_per_request;",
                                          lambda: tpa.test_per_request_filter_equals_separate_calls("topk_first")),
    "verify reads the first request's params": (
        "p_cnt[i] = filter_row(row, dtype, vocab, sp_T(sp, r), sp_k(sp, r), sp_p(sp, r), sp->order,",
        "p_cnt[i] = filter_row(row, dtype, vocab, sp_T(sp, 0), sp_k(sp, 0), sp_p(sp, 0), sp->order,",
        lambda: tpa.test_per_request_linear_verify_equals_separate_calls("joint")),
    "cycle verifies against the same-index target row": (
        "const int32_t* pi_ids = p_ids + (size_t)(i - 1) * (size_t)cap;\n                const float* pi_pr = p_pr + (size_t)(i - 1) * (size_t)cap;",
        "const int32_t* pi_ids = p_ids + (size_t)i * (size_t)cap;\n                const float* pi_pr = p_pr + (size_t)i * (size_t)cap;",
        lambda: tc.test_cycle_equals_generic_form_with_a_certain_first_draft(4, "topk_first", False)),
    "cycle bonus from the first target row": (
        "const int32_t* pb_ids = p_ids + (size_t)(B - 1) * (size_t)cap;\n                const float* pb_pr = p_pr + (size_t)(B - 1) * (size_t)cap;",
        "const int32_t* pb_ids = p_ids;\n                const float* pb_pr = p_pr;",
        lambda: tc.test_cycle_equals_generic_form_with_a_certain_first_draft(4, "topk_first", False)),
    "cycle counts the bonus as a correct draft": (
        "toks[B] = pick >= 0 ? pb_ids[pick] : -1;\n                ++emitted;",
        "toks[B] = pick >= 0 ? pb_ids[pick] : -1;\n                ++emitted;\n                ++correct;",
        tc.test_cycle_counters_and_output_slots),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(name, tmp_path):
    old, new, pin = MUTATIONS[name]
    assert SRC.count(old) == 1, f"mutation anchor for {name!r} not unique"
    src = tmp_path / "uno_ref_mut.c"
    src.write_text(SRC.replace(old, new))
    so = tmp_path / "libuno_ref_mut.so"
    subprocess.run(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-o", str(so), str(src), "-lm"], check=True)
    with oracle.use_library(so):
        with pytest.raises(AssertionError):
            pin()
