"""Planted mistakes: each case edits one spot of the oracle's C source (a dropped term, a wrong sign
or index, a swapped operand, an off-by-one), compiles the edited copy into a scratch library and
runs the pins that should notice.  Every case must make at least one of its pins fail, which shows
the pins constrain that spot; the unedited oracle passes the same pins in test_oracle_pins.py.

Only the oracle is edited, on the CPU, in a temporary directory; the committed source stays as it
is.  Edits are chosen so that the edited program stays inside its buffers.
"""
import os

import pytest

import oracle
from oracle import _build

from . import test_oracle_pins as P

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")

# (name, exact text in oracle.c, replacement, [(pin, args), ...])
MUTANTS = [
    # tree ancestry
    ("ancestry_parent_bit_only",
     "anc[i] = anc[p] | (1ull << i);", "anc[i] = (1ull << p) | (1ull << i);",
     [(P.test_ancestry_equals_transitive_closure, ())]),
    ("ancestry_root_not_its_own_ancestor",
     "anc[0] = 1ull;", "anc[0] = 0ull;",
     [(P.test_ancestry_equals_transitive_closure, ())]),
    ("ancestry_depth_not_advanced",
     "depth[i] = depth[p] + 1;", "depth[i] = depth[p];",
     [(P.test_ancestry_equals_transitive_closure, ())]),
    # attention
    ("attention_mask_by_index_order",
     "if (!((anc[i] >> j) & 1ull)) { s[L + j] = -INFINITY; continue; }",
     "if (j > i) { s[L + j] = -INFINITY; continue; }",
     [(P.test_tree_attention_equals_dense_closure_mask, (16, 6, 4, None))]),
    ("attention_cache_scores_unscaled",
     "                s[t] = scale * acc;\n", "                s[t] = acc;\n",
     [(P.test_chain_tree_equals_causal_attention, ())]),
    ("attention_gqa_heads_round_robin",
     "int kvh = h / group;", "int kvh = h % hkv;",
     [(P.test_tree_attention_equals_dense_closure_mask, (16, 6, 4, None))]),
    ("attention_cache_rows_ignore_slot_base",
     "const uint16_t *kr = k_cache + ((size_t)(slot_base[r] + t) * hkv + kvh) * d;",
     "const uint16_t *kr = k_cache + ((size_t)(t) * hkv + kvh) * d;",
     [(P.test_single_node_tree_equals_one_token_decode, ())]),
    ("attention_tree_values_read_from_keys",
     ": v_tree + ((size_t)(base + (t - L)) * hkv + kvh) * d;",
     ": k_tree + ((size_t)(base + (t - L)) * hkv + kvh) * d;",
     [(P.test_chain_tree_equals_causal_attention, ())]),
    ("attention_lse_without_max",
     "if (lse) lse[k] = mx + log(den);", "if (lse) lse[k] = log(den);",
     [(P.test_chain_tree_equals_causal_attention, ())]),
    # LM head
    ("logits_weight_transposed",
     "wrow[h] = bf16_value(w[(size_t)v * H + h]);", "wrow[h] = bf16_value(w[(size_t)h * V + v]);",
     [(P.test_logits_equal_numpy_matmul, ())]),
    ("argmax_ties_to_highest_id",
     "if (row[v] > row[best]) best = v;", "if (row[v] >= row[best]) best = v;",
     [(P.test_row_top2_ties_and_order, ())]),
    ("top2_skips_a_repeated_maximum",
     "if (v != best && row[v] > second) second = row[v];",
     "if (row[v] != row[best] && row[v] > second) second = row[v];",
     [(P.test_row_top2_ties_and_order, ())]),
    # greedy walk
    ("greedy_highest_index_duplicate_child",
     "if (parent[c] == u && tokens[c] == want) { next = c; break; }",
     "if (parent[c] == u && tokens[c] == want) { next = c; }",
     [(P.test_greedy_walk_duplicate_siblings_take_the_lowest_index, ())]),
    ("greedy_bonus_from_the_root",
     "    out_tokens[a] = arg[u];\n    return a;", "    out_tokens[a] = arg[0];\n    return a;",
     [(P.test_greedy_walk_equals_sequential_greedy_decoding, (s,)) for s in range(12)]),
    # Philox and the uniforms
    ("philox_key_words_swapped",
     "uint64_t n0 = hi1 ^ c1 ^ k0, n1 = lo1, n2 = hi0 ^ c3 ^ k1, n3 = lo0;",
     "uint64_t n0 = hi1 ^ c1 ^ k1, n1 = lo1, n2 = hi0 ^ c3 ^ k0, n3 = lo0;",
     [(P.test_philox_random_counters_match_numpy, ())]),
    ("philox_weyl_constant",
     "W1 = 0xBB67AE8584CAA73Bull", "W1 = 0xBB67AE8584CAA73Aull",
     [(P.test_philox_random_counters_match_numpy, ())]),
    ("philox_nine_rounds",
     "for (int round = 0; round < 10; ++round)", "for (int round = 0; round < 9; ++round)",
     [(P.test_philox_random_counters_match_numpy, ())]),
    ("uniform_field_too_wide",
     ": (x >> 41);", ": (x >> 40);",
     [(P.test_uniform_is_23bit_centred_exact_in_float32_and_uniform, ())]),
    ("uniform_not_centred",
     "return ((double)field + 0.5) * (1.0 / 8388608.0);",
     "return ((double)field) * (1.0 / 8388608.0);",
     [(P.test_uniform_is_23bit_centred_exact_in_float32_and_uniform, ())]),
    # samplers
    ("race_gumbel_sign",
     "double key = log(w[v]) - log(-log(U));", "double key = log(w[v]) + log(-log(U));",
     [(P.test_exponential_race_is_an_exact_sampler, ())]),
    ("race_ignores_the_weights",
     "double key = log(w[v]) - log(-log(U));", "double key = -log(-log(U));",
     [(P.test_exponential_race_is_an_exact_sampler, ())]),
    ("chain_fallback_takes_the_mode_of_p",
     "            fell_back = 1;\n            bonus = oracle_race(V, p, seed, step, r, u, NULL);",
     "            fell_back = 1;\n            bonus = 0;\n"
     "            for (int v = 1; v < V; ++v) if (p[v] > p[bonus]) bonus = v;",
     [(P.test_empty_residual_draws_the_bonus_from_the_target, ())]),
    ("tree_fallback_returns_a_fixed_token",
     "    if (fell_back) bonus = oracle_race(V, p, seed, step, r, u, NULL);",
     "    if (fell_back) bonus = 0;",
     [(P.test_empty_residual_draws_the_bonus_from_the_target, ())]),
    # stochastic acceptance on chains
    ("chain_test_p_and_q_swapped",
     "if (U * qx < p[x]) {", "if (U * p[x] < qx) {",
     [(P.test_first_emitted_token_follows_target, (1.0,))]),
    ("chain_residual_without_q",
     "double d = p[v] - (double)q[(size_t)u * V + v];", "double d = p[v];",
     [(P.test_rejected_draft_residual_excludes_the_rejected_token_mass, ())]),
    ("chain_bonus_at_the_root",
     "int u = a;  /* stop node", "int u = 0;  /* stop node",
     [(P.test_second_emitted_token_follows_target_given_accepted_prefix, ())]),
    ("softmax_drops_the_temperature",
     "for (int v = 0; v < V; ++v) p[v] = exp(z[v] / T - lse);",
     "for (int v = 0; v < V; ++v) p[v] = exp(z[v] - lse);",
     [(P.test_first_emitted_token_follows_target, (0.7,))]),
    # stochastic acceptance on branching trees
    ("tree_residual_not_renormalised",
     "rx = rx > 0.0 ? rx / Nc : 0.0;", "rx = rx > 0.0 ? rx : 0.0;",
     [(P.test_multi_candidate_first_token_follows_target, (2, 1.0))]),
    ("tree_scale_advanced_by_one",
     "            c += Nc;\n", "            c += 1.0;\n",
     [(P.test_multi_candidate_first_token_follows_target, (2, 1.0))]),
    ("tree_siblings_share_one_uniform",
     "oracle_uniform(seed, step, (uint32_t)r, (uint32_t)j, 0, 1);",
     "oracle_uniform(seed, step, (uint32_t)r, (uint32_t)u + 1u, 0, 1);",
     [(P.test_multi_candidate_sibling_acceptance_rates_match_the_closed_form, ())]),
    ("tree_bonus_ignores_rejections",
     "            const double d = p[v] - c * (double)qu[v];\n"
     "            w[v] = d > 0.0 ? d : 0.0;",
     "            const double d = p[v] + 0.0 * c * (double)qu[v];\n"
     "            w[v] = d > 0.0 ? d : 0.0;",
     [(P.test_multi_candidate_residual_excludes_rejected_mass, ())]),
    # compaction
    ("compact_destination_ignores_kv_len",
     "+ (size_t)(slot_base[r] + kv_len[r] + k) * row;", "+ (size_t)(slot_base[r] + k) * row;",
     [(P.test_kv_compact_equals_numpy_gather, ())]),
    ("compact_new_length_misses_the_root",
     "kv_len_out[r] = kv_len[r] + a + 1;\n    }", "kv_len_out[r] = kv_len[r] + a;\n    }",
     [(P.test_kv_compact_equals_numpy_gather, ())]),
    ("compact_capacity_off_by_one",
     "if ((int64_t)kv_len[r] + a + 1 > (int64_t)slot_cap[r])",
     "if ((int64_t)kv_len[r] + a > (int64_t)slot_cap[r])",
     [(P.test_kv_compact_fills_capacity_exactly_and_no_further, ())]),
    ("compact_source_row_from_path_index",
     "size_t src = (size_t)l * tree_layer_stride + (size_t)(cu_nodes[r] + j) * row;",
     "size_t src = (size_t)l * tree_layer_stride + (size_t)(cu_nodes[r] + k) * row;",
     [(P.test_kv_compact_equals_numpy_gather, ())]),
    ("compact_first_layer_only",
     "        for (int l = 0; l < n_layers; ++l)\n", "        for (int l = 0; l < 1; ++l)\n",
     [(P.test_kv_compact_equals_numpy_gather, ())]),
    ("greedy_accepts_any_child",
     "if (parent[c] == u && tokens[c] == want) { next = c; break; }",
     "if (parent[c] == u) { next = c; break; }",
     [(P.test_greedy_walk_equals_sequential_greedy_decoding, (s,)) for s in range(12)]),
    ("tree_keeps_testing_siblings_after_an_accept",
     "                next = j;\n                break;", "                next = j;",
     [(P.test_multi_candidate_sibling_acceptance_rates_match_the_closed_form, ())]),
    ("attention_last_tree_key_left_out_of_the_sum",
     "for (long t = 0; t < nkeys; ++t) {", "for (long t = 0; t < nkeys - 1; ++t) {",
     [(P.test_chain_tree_equals_causal_attention, ())]),
    # bf16 rounding and the low-rank head
    ("bf16_ties_away_from_zero",
     "else r = fmod(lo / ulp, 2.0) == 0.0 ? lo : hi;", "else r = hi;",
     [(P.test_bf16_rounding_is_nearest_even, ())]),
    ("lowrank_down_projection_rounded_to_bf16",
     "        g[t] = acc;\n", "        g[t] = bf16_value(oracle_bf16_round(acc));\n",
     [(P.test_lowrank_screen_is_the_factorised_product, ())]),
    ("lowrank_screen_ties_to_highest_id",
     "if (!taken[v] && (best < 0 || z[v] > z[best])) best = v;",
     "if (!taken[v] && (best < 0 || z[v] >= z[best])) best = v;",
     [(P.test_lowrank_screen_is_the_factorised_product, ())]),
    ("lowrank_kth_is_the_best_screen_value",
     "if (kth) kth[m] = z[cand[k - 1]];", "if (kth) kth[m] = z[cand[0]];",
     [(P.test_lowrank_screen_is_the_factorised_product, ())]),
    ("lowrank_exact_order_ascending",
     "while (j >= 0 && (ex[j] < xi || (ex[j] == xi && cand[j] > ci))) {",
     "while (j >= 0 && (ex[j] > xi || (ex[j] == xi && cand[j] > ci))) {",
     [(P.test_lowrank_head_with_identity_factors_is_the_exact_top_k, ())]),
]


def _source():
    with open(_build.SRC) as f:
        return f.read()


def test_every_planted_spot_exists_once():
    src = _source()
    for name, old, new, _ in MUTANTS:
        assert src.count(old) == 1, name
        assert old != new, name
    assert len({m[0] for m in MUTANTS}) == len(MUTANTS)


@pytest.mark.parametrize("name,old,new,pins", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_the_planted_mistake(name, old, new, pins, tmp_path, monkeypatch):
    src = _source()
    assert src.count(old) == 1
    c_path = os.path.join(tmp_path, "mutant.c")
    with open(c_path, "w") as f:
        f.write(src.replace(old, new))
    lib_path = _build.compile_to(c_path, os.path.join(tmp_path, "libmutant.so"))
    monkeypatch.setattr(oracle, "_lib", oracle._bind(lib_path))
    caught = []
    for pin, args in pins:
        try:
            pin(*args)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"{name}: no pin failed"


# The paged forms are numpy compositions in oracle/__init__.py: each case edits one function's
# source text, rebinds the edited function in the oracle module and runs the paged pins.
PY_MUTANTS = [
    ("page_slots_offset_in_page_dropped", "page_slots",
     "[r, t // page_size].astype(np.int64) * page_size + t % page_size",
     "[r, t // page_size].astype(np.int64) * page_size",
     [(P.test_page_slots_by_hand, ())]),
    ("paged_attention_every_request_at_offset_zero", "attention_paged",
     "        base[r] = off\n", "        base[r] = 0\n",
     [(P.test_paged_attention_is_independent_of_page_placement, ())]),
    ("paged_compaction_writes_from_position_zero", "kv_compact_paged",
     "np.arange(L, L + a + 1))", "np.arange(0, a + 1))",
     [(P.test_paged_compaction_equals_contiguous_compaction_of_the_logical_cache, ())]),
    ("paged_compaction_source_ignores_request_offset", "kv_compact_paged",
     "src = int(cu[r]) + pr", "src = pr",
     [(P.test_paged_compaction_equals_contiguous_compaction_of_the_logical_cache, ())]),
]


def test_every_planted_python_spot_exists_once():
    import inspect
    for name, fn, old, new, _ in PY_MUTANTS:
        assert inspect.getsource(getattr(oracle, fn)).count(old) == 1, name
        assert old != new, name


@pytest.mark.parametrize("name,fn,old,new,pins", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_pins_catch_the_planted_python_mistake(name, fn, old, new, pins, monkeypatch):
    import inspect
    src = inspect.getsource(getattr(oracle, fn))
    assert src.count(old) == 1
    scope = dict(vars(oracle))
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), scope)
    monkeypatch.setattr(oracle, fn, scope[fn])
    caught = []
    for pin, args in pins:
        try:
            pin(*args)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"{name}: no pin failed"
