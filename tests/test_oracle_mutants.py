"""The oracle's pins catch plausible mistakes (CPU only).

Each case plants one mistake in a private copy of oracle.c (a flipped tie
break, an off-by-one in the quota remainder, a loosened stop test, a wrong
index...), builds it, and runs the pin tests against it: at least one pin
must fail. The real oracle is never modified.
"""
import ctypes
import os
import subprocess
import sys

import pytest

import oracle
from tests import test_oracle_gate as tg
from tests import test_oracle_plan as tp
from tests import test_oracle_backward as tb
from tests import test_oracle_rows as tr
from tests import test_oracle_variants as tv

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "topk_tie_to_higher_id": ("if (a->e < b->e) return -1;\n    if (a->e > b->e) return 1;",
                              "if (a->e < b->e) return 1;\n    if (a->e > b->e) return -1;"),
    "topk_signed_zero_not_tied": (
        "if (a->v > b->v) return -1;\n    if (a->v < b->v) return 1;",
        "if (a->v > b->v || (a->v == b->v && signbit(b->v) && !signbit(a->v))) return -1;\n"
        "    if (a->v < b->v || (a->v == b->v && signbit(a->v) && !signbit(b->v))) return 1;"),
    "topk_weight_unshifted": ("w[n * K + k] = exp((double)row[k].v - v0) / z;",
                              "w[n * K + k] = exp((double)row[k].v) / z;"),
    "count_rank_from_pair": ("int64_t r = n / T;", "int64_t r = i / T;"),
    "quota_remainder_off_by_one": ("return L / c + (j < L % c ? 1 : 0);",
                                   "return L / c + (j <= L % c ? 1 : 0);"),
    "stop_strict": ("if (50 * (int64_t)R * maxl <= 51 * Q) break;",
                    "if (50 * (int64_t)R * maxl < 51 * Q) break;"),
    "stop_looser": ("if (50 * (int64_t)R * maxl <= 51 * Q) break;",
                    "if (50 * (int64_t)R * maxl <= 52 * Q) break;"),
    "rank_tie_to_higher_r": ("if (used < S && (rstar < 0 || load[r] < load[rstar])) rstar = r;",
                             "if (used < S && (rstar < 0 || load[r] <= load[rstar])) rstar = r;"),
    "expert_tie_to_higher_e": ("(int64_t)load_e[e] * n_copies[estar] >\n",
                               "(int64_t)load_e[e] * n_copies[estar] >=\n"),
    "remainder_by_descending_slot": ("for (int32_t g = 0; g < G; ++g) {\n            if (slot_expert[g] == e) {\n                load[g / S]",
                                     "for (int32_t g = G - 1; g >= 0; --g) {\n            if (slot_expert[g] == e) {\n                load[g / S]"),
    "reroute_row_without_start": ("dest_row[i] = slot_offset[found] + (int32_t)(o - start);",
                                  "dest_row[i] = slot_offset[found] + (int32_t)o;"),
    "permute_wrong_token": ("memcpy(dispatch + row * d, hidden + (i / K) * d,",
                            "memcpy(dispatch + row * d, hidden + (i % K) * d,"),
    "combine_first_weight_only": ("double wk = w[n * K + k];", "double wk = w[n * K];"),
    "backward_dy_without_weight": ("dy_rows[(j * K + k) * d + c] = wk * g;",
                                   "dy_rows[(j * K + k) * d + c] = g;"),
    "backward_dw_wrong_row": ("dot += g * or_bf16_to_double(y[row * d + c]);",
                              "dot += g * or_bf16_to_double(y[(n * K) * d + c]);"),
    "permute_backward_drops_last_k": ("        for (int32_t k = 0; k < K; ++k) {\n            int64_t row = dest_row[n * K + k];\n            if (row < 0 || row >= Q) return OR_EDATA;\n            for (int32_t c = 0; c < d; ++c)\n                dhidden",
                                      "        for (int32_t k = 0; k + 1 < K; ++k) {\n            int64_t row = dest_row[n * K + k];\n            if (row < 0 || row >= Q) return OR_EDATA;\n            for (int32_t c = 0; c < d; ++c)\n                dhidden"),
    "weight_sync_wrong_source": ("memcpy(replicas + (int64_t)g * bytes_per_expert, master + (int64_t)e * bytes_per_expert,",
                                 "memcpy(replicas + (int64_t)g * bytes_per_expert, master + (int64_t)g % E * bytes_per_expert,"),
    "greedy_minimum_without_new_copy": ("if ((int64_t)load_e[e] < (int64_t)min_tokens * (n_copies[e] + 1)) continue;",
                                        "if ((int64_t)load_e[e] < (int64_t)min_tokens * n_copies[e]) continue;"),
    "bisect_shed_smallest_master_first": ("if (!done[e] && (best < 0 || L[e] > L[best])) best = e;",
                                          "if (!done[e] && (best < 0 || L[e] < L[best])) best = e;"),
    "bisect_no_raise_to_minimum": ("if (s < m) s = m;", ";"),
    "bisect_no_cut_rule": ("if (rem - piece > 0 && rem - piece < m) piece = rem - m;", ";"),
    "bisect_receiver_tie_to_higher_r": ("if (rs < 0 || spare[r] > spare[rs]) rs = r;",
                                        "if (rs < 0 || spare[r] >= spare[rs]) rs = r;"),
    "bisect_smallest_demand_first": ("if (!done[f] && shed[f] > 0 && (e < 0 || shed[f] > shed[e])) e = f;",
                                     "if (!done[f] && shed[f] > 0 && (e < 0 || shed[f] < shed[e])) e = f;"),
    "bisect_mid_rounds_up": ("int64_t mid = lo + (hi - lo) / 2;", "int64_t mid = lo + (hi - lo + 1) / 2;"),
    "bisect_capacity_rounds_up": ("int rc = or_quota_oracle(R, E, S, load_e, k * Q / DR,",
                                  "int rc = or_quota_oracle(R, E, S, load_e, (k * Q + DR - 1) / DR,"),
    "bisect_master_may_always_empty": ("int64_t keep = (allow_zero || L[best] == 0) ? 0 : 1;",
                                       "int64_t keep = 0;"),
    "split_without_local_pass": ("int64_t a = s[h] < q[j] ? s[h] : q[j];", "int64_t a = 0;"),
    "split_remote_descending": ("for (int32_t r = 0; r < R && q[j] > 0; ++r) {",
                                "for (int32_t r = R - 1; r >= 0 && q[j] > 0; --r) {"),
    "interleave_rank_major": ("    for (int32_t t = 0; t < T; ++t) {\n        for (int32_t r = 0; r < R; ++r) {",
                              "    for (int32_t r = 0; r < R; ++r) {\n        for (int32_t t = 0; t < T; ++t) {"),
    "local_row_without_source_offset": ("dest_row[i] = src_offset[(int64_t)r * P + found] + (int32_t)(o - start);",
                                        "dest_row[i] = src_offset[found] + (int32_t)(o - start);"),
    "greedy_needs_a_pair_per_copy": ("if ((int64_t)load_e[e] < (int64_t)min_tokens * (n_copies[e] + 1)) continue;",
                                     "if ((int64_t)load_e[e] < (int64_t)(min_tokens > 0 ? min_tokens : 1) * (n_copies[e] + 1)) continue;"),
    "colocation_counts_masters_only": ("        for (int32_t s = 0; s < S; ++s)\n            if (slot_expert[rstar * S + s] == estar) hosts = 1;\n",
                                       ""),
    "reroute_replica_end_inclusive": ("if (o < start + slot_quota[p]) found = p;",
                                      "if (o <= start + slot_quota[p]) found = p;"),
    "topk_softmax_over_k_plus_one": ("for (int32_t k = 0; k < K; ++k) z += exp((double)row[k].v - v0);",
                                     "for (int32_t k = 0; k <= K && k < E; ++k) z += exp((double)row[k].v - v0);"),
    "combine_drops_last_k": ("out[j * d + c] = 0.0;\n        for (int32_t k = 0; k < K; ++k) {",
                             "out[j * d + c] = 0.0;\n        for (int32_t k = 0; k + 1 < K; ++k) {"),
    "grad_reduce_skips_master": ("out[(int64_t)e * numel + i] = (double)master[(int64_t)e * numel + i];",
                                 "out[(int64_t)e * numel + i] = 0.0;"),
}


def run_pins(golden_dir):
    """Every pin of the oracle; returns the names of those that failed."""
    pins = [
        ("hand_row", tg.test_hand_row_closed_form),
        ("signed_zero", tg.test_signed_zero_ties_to_lower_id),
        ("all_equal", tg.test_all_equal_rows_pick_lowest_ids_and_uniform_weights),
        ("brute_topk", lambda: tg.test_matches_brute_force_with_many_ties(64, 4)),
        ("softmax", lambda: tg.test_weights_equal_renormalised_full_softmax(128, 8)),
        ("count_uniform", tg.test_count_constructed_uniform_routing),
        ("count_random", tg.test_count_random_matches_bincount),
        ("hand_plans", lambda: tp.test_hand_worked_plans(golden_dir)),
        ("plan_invariants", lambda: tp.test_plan_invariants_random(8, 64, 2, 1.2)),
        ("plan_hot", tp.test_plan_single_hot_expert_closed_form),
        ("plan_unbalanceable", tp.test_plan_that_cannot_balance_places_zero_quota_copies),
        ("hand_reroute", lambda: tp.test_reroute_hand_worked(golden_dir)),
        ("reroute_invariants", lambda: tp.test_reroute_invariants_random(4, 33, 16, 3, 2)),
        ("reroute_zero_quota", lambda: tp.test_reroute_with_zero_quota_copies(4, 8, 4, 3)),
        ("permute", tr.test_permute_definition_small),
        ("combine_exact", tr.test_combine_exact_dyadic_case),
        ("combine_identity", tr.test_combine_identity_experts_reproduce_hidden),
        ("bwd_hand", tb.test_combine_backward_hand_case),
        ("bwd_adjoint", tb.test_combine_backward_adjoint_identities),
        ("pbwd_adjoint", tb.test_permute_backward_adjoint_identity),
        ("pbwd_hand", tb.test_permute_backward_sums_k_rows),
        ("wsync", tb.test_weight_sync_definition),
        ("greduce_hand", tb.test_grad_reduce_dyadic_hand_case),
        ("greduce_np", tb.test_grad_reduce_matches_numpy_add_at),
        ("bisect_hand", lambda: tv.test_bisect_hand_cases(golden_dir)),
        ("greedy_min_hand", lambda: tv.test_greedy_min_tokens_hand_cases(golden_dir)),
        ("split_hand", lambda: tv.test_locality_split_hand_cases(golden_dir)),
        ("bisect_invariants", lambda: tv.test_bisect_invariants_random(8, 64, 2, 1.2, 16)),
        ("bisect_opt", lambda: tv.test_bisect_bounded_by_exhaustive_opt(2, 4, 1)),
        ("greedy_min_invariants", lambda: tv.test_greedy_min_tokens_invariants(8, 64, 2, 1.2, 64)),
        ("split_invariants", lambda: tv.test_locality_split_invariants(8, 128, 64, 4, 2, True, "greedy")),
        ("split_remote", lambda: tv.test_locality_cuts_remote_pairs_of_a_hot_expert(golden_dir)),
        ("interleave", lambda: tv.test_interleave_is_prefix_fill_in_token_major_order(8, 128, 64, 4, 2, "greedy")),
    ]
    failed = []
    for name, fn in pins:
        try:
            fn()
        except (AssertionError, ValueError):
            failed.append(name)
    return failed


def test_real_oracle_passes_every_pin(golden_dir):
    assert run_pins(golden_dir) == []


_CHILD = """
import ctypes, sys
sys.path.insert(0, {root!r})
import oracle
from tests import test_oracle_mutants as m
oracle._lib = oracle._bind(ctypes.CDLL({so!r}))
failed = m.run_pins({golden!r})
print("FAILED_PINS", failed)
sys.exit(1 if failed else 0)
"""


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, golden_dir, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fPIC",
                           "-shared", "-o", str(so), str(path), "-lm"])
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    # a child process, so that a mutant that writes out of bounds and crashes
    # (which also counts as caught) cannot take the test run down with it
    res = subprocess.run([sys.executable, "-c",
                          _CHILD.format(root=root, so=str(so), golden=golden_dir)],
                         capture_output=True, text=True, timeout=300)
    assert res.returncode != 0, f"no pin caught the planted mistake '{name}':\n{res.stdout}"
