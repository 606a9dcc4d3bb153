"""Plants plausible mistakes in the oracle (CPU only, via monkeypatch) and checks that at least one pin
fails for each, so the pins are known to bite."""
import numpy as np

import importlib

acc_mod = importlib.import_module("oracle.accept")
bt_mod = importlib.import_module("oracle.build_tree")
ta_mod = importlib.import_module("oracle.tree_attention")
fr_mod = importlib.import_module("oracle.frontier")
from tests import test_oracle_accept as TA
from tests import test_oracle_frontier as TFR
from tests import test_oracle_attention as TT
from tests import test_oracle_build as TB


def fails(fn, *a):
    try:
        fn(*a)
    except (AssertionError, ValueError, IndexError):
        return True
    return False


def test_dropping_self_is_caught(monkeypatch):
    def anc_no_self(parent):
        anc = []
        for i, p in enumerate(parent.tolist()):
            base = (anc[p] | {p}) if p >= 0 else set()
            anc.append(base)
        return anc
    monkeypatch.setattr(ta_mod, "ancestor_sets", anc_no_self)
    assert fails(TT.test_star_equals_prefix_plus_self)


def test_seeing_siblings_is_caught(monkeypatch):
    orig = ta_mod.ancestor_sets

    def anc_with_siblings(parent):
        anc = orig(parent)
        for i, p in enumerate(parent.tolist()):
            anc[i] = anc[i] | {j for j in range(len(parent)) if parent[j] == p and p >= 0}
        return anc
    monkeypatch.setattr(ta_mod, "ancestor_sets", anc_with_siblings)
    assert fails(TT.test_path_extraction_branch_factorisation, 4)


def test_transposed_page_index_is_caught(monkeypatch):
    def bad_gather(cache, block_row, slots, kv_head):
        return cache[block_row[slots % 16 % len(block_row)], slots // 16 % 16, kv_head, :].astype(np.float64)
    monkeypatch.setattr(ta_mod, "gather_slots", bad_gather)
    assert fails(TT.test_chain_equals_causal_attention)


def test_wrong_gqa_map_is_caught(monkeypatch):
    orig = ta_mod.gather_slots
    monkeypatch.setattr(ta_mod, "gather_slots", lambda c, r, s, h: orig(c, r, s, (h + 1) % c.shape[2]))
    assert fails(TT.test_chain_equals_causal_attention)


def test_wrong_depth_row_is_caught(monkeypatch):
    orig = bt_mod.row_stats
    calls = {"n": 0}

    def shifted_stats(x):  # pretend the normaliser of each row were off by a depth-dependent amount
        calls["n"] += 1
        m, lse = orig(x)
        return m, lse + 0.01 * calls["n"]
    monkeypatch.setattr(bt_mod, "row_stats", shifted_stats)
    assert fails(TB.test_brute_force_full_tree, 2, 3, 4, 40)


def test_sibling_order_is_caught(monkeypatch):
    monkeypatch.setattr(bt_mod, "topk_tokens", lambda x, k: np.argsort(np.asarray(x))[:k])
    assert fails(TB.test_topk1_is_chain_of_argmaxes)


def test_highest_id_tie_break_is_caught(monkeypatch):
    def last_argmax(row):
        row = np.asarray(row)
        return len(row) - 1 - int(np.argmax(row[::-1]))
    monkeypatch.setattr(acc_mod, "first_argmax", last_argmax)
    assert fails(TA.test_argmax_ties_take_lowest_id)


ck_mod = importlib.import_module("oracle.commit_kv")
from tests import test_oracle_commit as TC


def test_commit_ignoring_the_block_table_is_caught(monkeypatch):
    monkeypatch.setattr(ck_mod, "locate", lambda row, s: (s // 16, s % 16))
    assert fails(TC.test_hand_worked_example)


def test_commit_slots_off_by_one_is_caught(monkeypatch):
    real = ck_mod.commit_kv

    def off_by_one(k_cache, v_cache, bt, prefix, offs, path, L):
        return real(k_cache, v_cache, bt, [int(p) - 1 if int(p) > 0 else 0 for p in prefix], offs, path, L)
    monkeypatch.setattr(TC, "commit_kv", off_by_one)
    assert fails(TC.test_hand_worked_example)


def test_commit_in_place_in_reverse_order_is_caught(monkeypatch):
    def reverse_in_place(k_cache, v_cache, block_table, prefix_lens, tree_offsets, path, accepted_len):
        k, v = np.array(k_cache, copy=True), np.array(v_cache, copy=True)
        newp = np.array(prefix_lens, dtype=np.int64).copy()
        for b in range(len(prefix_lens)):
            P, N, L = int(prefix_lens[b]), int(tree_offsets[b + 1]) - int(tree_offsets[b]), int(accepted_len[b])
            if N == 0:
                continue
            for i in range(L, 0, -1):  # no staging, last copy first
                ps, os_ = ck_mod.locate(block_table[b], P + int(path[b][i]))
                pd, od = ck_mod.locate(block_table[b], P + i)
                k[pd, od], v[pd, od] = k[ps, os_].copy(), v[ps, os_].copy()
            newp[b] = P + L + 1
        return k, v, newp.astype(np.int32)
    monkeypatch.setattr(TC, "commit_kv", reverse_in_place)
    assert fails(TC.test_sources_that_are_later_destinations)


ka_mod = importlib.import_module("oracle.kv_append")
from tests import test_oracle_kv_append as TK


def test_rope_interleaved_pairs_are_caught(monkeypatch):
    def interleaved(x, pos, theta):
        x = np.asarray(x, dtype=np.float64)
        d = x.shape[-1]
        inv = np.power(float(theta), -2.0 * np.arange(d // 2, dtype=np.float64) / d)
        ang = np.asarray(pos, dtype=np.float64)[..., None] * inv
        c, s = np.cos(ang), np.sin(ang)
        out = x.copy()
        out[..., 0::2] = x[..., 0::2] * c - x[..., 1::2] * s
        out[..., 1::2] = x[..., 1::2] * c + x[..., 0::2] * s
        return out
    monkeypatch.setattr(TK, "rope", interleaved)
    assert fails(TK.test_hand_worked_d4)


def test_rope_position_off_by_one_is_caught(monkeypatch):
    orig = ka_mod.node_positions
    monkeypatch.setattr(ka_mod, "node_positions", lambda p, o, d: orig(p, o, d) - 1)
    assert fails(TK.test_nodes_land_in_their_slots_with_their_positions)


def test_rope_wrong_frequency_base_is_caught(monkeypatch):
    orig = ka_mod.rope
    monkeypatch.setattr(TK, "rope", lambda x, pos, theta: orig(x, pos, theta * 10))
    assert fails(TK.test_matches_complex_formulation, 1e4)


fp8_mod = importlib.import_module("oracle.fp8_kv")
from tests import test_oracle_fp8 as TF


def test_e4m3_wrong_bias_is_caught(monkeypatch):
    orig = fp8_mod.e4m3_decode
    monkeypatch.setattr(TF, "e4m3_decode", lambda c: orig(c) * 2.0)
    assert fails(TF.test_all_codes_match_torch)


def test_e4m3_ties_away_from_zero_is_caught(monkeypatch):
    def away(x):
        x = np.asarray(x, dtype=np.float64)
        a = np.minimum(np.abs(x), 448.0)
        vals = fp8_mod._POS
        idx = np.array([int(np.argmin(np.abs(vals - v) - 1e-12 * (vals > v))) for v in a.ravel()]).reshape(a.shape)
        return np.where(np.signbit(x), idx | 0x80, idx).astype(np.uint8)
    monkeypatch.setattr(TF, "e4m3_encode", away)
    assert fails(TF.test_round_trip_and_ties_to_even)


def test_e4m3_no_saturation_is_caught(monkeypatch):
    orig = fp8_mod.e4m3_encode
    monkeypatch.setattr(TF, "e4m3_encode", lambda x: np.where(np.abs(np.asarray(x, dtype=np.float64)) > 464.0, 0x7F,
                                                             orig(x)).astype(np.uint8))
    assert fails(TF.test_saturation)


def test_frontier_key_without_the_parent_score_is_caught(monkeypatch):
    monkeypatch.setattr(fr_mod, "candidate_key", lambda parent_key, lp: lp)
    assert fails(TFR.test_width_one_with_path_conditioned_rows_is_exact_best_first, 11, 2, 4, 20)


def test_frontier_reoffering_taken_children_is_caught(monkeypatch):
    monkeypatch.setattr(fr_mod, "untaken", lambda state, u: range(len(state.cand_tok[u])))
    assert fails(TFR.test_invariants, 7)


def test_frontier_lp_without_the_normaliser_is_caught(monkeypatch):
    def children_no_lse(row, topk):
        row = np.asarray(row)
        tok = fr_mod.topk_tokens(row, topk)
        return tok, row[tok].astype(np.float64)
    monkeypatch.setattr(fr_mod, "node_children", children_no_lse)
    assert fails(TFR.test_invariants, 3)


def test_frontier_children_of_this_rounds_picks_are_caught(monkeypatch):
    # a round that scores every node it adds at once (as if its row were already known) loses the round structure:
    # children join in the same round as their parent
    orig = fr_mod.expand_frontier

    def eager(state, rows, root_token, topk, max_depth, width):
        added = orig(state, rows, root_token, topk, max_depth, 1)
        while added < width and state.num_nodes < state.budget:
            fr_mod.start_tree(state, root_token)
            new = list(state.frontier())
            extra = [TFR.synth.path_logits(31 + width, state.path_tokens(i), 500) for i in new]
            a = orig(state, extra, root_token, topk, max_depth, 1)
            if a == 0:
                break
            added += a
        return added
    monkeypatch.setattr(fr_mod, "expand_frontier", eager)
    assert fails(TFR.test_invariants, 7)
