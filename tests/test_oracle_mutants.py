"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins catch each.

Each mutant replaces one oracle function with a subtly wrong version: a dropped term, a
wrong sign or index, an off-by-one, a transposed operand.  The pin named beside it must
then fail.  This shows the pins constrain the oracle, not just exercise it.
"""
import numpy as np
import pytest

import oracle as O
import oracle.dsa_oracle as OD
import tests.test_oracle_pins as P


def _scores_no_relu(q_t, w_t, k, pos, pool=1):
    S = k.shape[0]; n = min(S, pos // pool + 1)
    out = np.full(S, -np.inf, dtype=np.float32)
    out[:n] = ((k[:n] @ q_t.T) @ np.asarray(w_t, np.float64)).astype(np.float32)
    return out


def _scores_excl_self(q_t, w_t, k, pos, pool=1):
    out = OD._orig["index_scores_row"](q_t, w_t, k, pos, pool)
    if pos // pool < k.shape[0]:
        out[pos // pool] = -np.inf
    return out


def _scores_weights_reversed(q_t, w_t, k, pos, pool=1):
    return OD._orig["index_scores_row"](q_t, np.asarray(w_t)[::-1].copy(), k, pos, pool)


def _scores_abs_instead_of_relu(q_t, w_t, k, pos, pool=1):
    S = k.shape[0]; n = min(S, pos // pool + 1)
    out = np.full(S, -np.inf, dtype=np.float32)
    out[:n] = (np.abs(k[:n] @ q_t.T) @ np.asarray(w_t, np.float64)).astype(np.float32)
    return out


def _topk_ties_high_index(scores, n_valid, k):
    n = int(min(n_valid, scores.shape[0])); out = np.full(k, -1, np.int32)
    order = np.lexsort((-np.arange(n), -np.asarray(scores[:n], np.float64)))
    out[: min(k, n)] = order[: min(k, n)]
    return out


def _topk_smallest(scores, n_valid, k):
    n = int(min(n_valid, scores.shape[0])); out = np.full(k, -1, np.int32)
    order = np.lexsort((np.arange(n), np.asarray(scores[:n], np.float64)))
    out[: min(k, n)] = order[: min(k, n)]
    return out


def _attn_no_scale(q_t, K, V, idx_row, sm_scale):
    return OD._orig["sparse_attn_row"](q_t, K, V, idx_row, 1.0)


def _attn_k_as_v(q_t, K, V, idx_row, sm_scale):
    return OD._orig["sparse_attn_row"](q_t, K, K[:, : V.shape[1]], idx_row, sm_scale)


def _attn_drop_last(q_t, K, V, idx_row, sm_scale):
    r = [i for i in idx_row if i >= 0]
    return OD._orig["sparse_attn_row"](q_t, K, V, np.array(r[:-1] if len(r) > 1 else r), sm_scale)


def _attn_dedup(q_t, K, V, idx_row, sm_scale):
    r = np.unique(np.asarray([i for i in idx_row if i >= 0], dtype=np.int64))
    return OD._orig["sparse_attn_row"](q_t, K, V, r if r.size else np.array([-1]), sm_scale)


def _decode_bias8(codes):
    v = OD._orig["e4m3_to_f64"](codes)
    c = np.asarray(codes, np.uint8)
    return np.where(((c >> 3) & 0xF) == 0, v, v / 2.0)


def _encode_truncate(x):
    x = np.asarray(x, np.float32)
    codes = OD._orig["f32_to_e4m3"](x)
    back = OD._orig["e4m3_to_f64"](codes)
    over = np.abs(back) > np.abs(x.astype(np.float64))
    return np.where(over & (codes & 0x7F > 0), codes - 1, codes).astype(np.uint8)


def _pool_half(k_idx, pool=4):
    kf = OD._orig["e4m3_to_f64"](k_idx).astype(np.float32)
    S = kf.shape[-2]; g = kf.reshape(kf.shape[:-2] + (S // 4, 4, kf.shape[-1]))
    return OD._orig["f32_to_e4m3"]((g[..., 0, :] + g[..., 1, :]) * np.float32(0.5))


def _pool_fixed_quarter(k_idx, pool=4):
    # the factor-4 scale kept for every factor: the mean of 2 or 8 keys comes out x2 or x0.5
    kf = OD._orig["e4m3_to_f64"](k_idx).astype(np.float32)
    S = kf.shape[-2]; g = kf.reshape(kf.shape[:-2] + (S // pool, pool, kf.shape[-1]))
    return OD._orig["f32_to_e4m3"](g.sum(axis=-2, dtype=np.float32) * np.float32(0.25))


def _pool_first_four_only(k_idx, pool=4):
    # a group of 8 pooled as if it held only its first 4 keys
    kf = OD._orig["e4m3_to_f64"](k_idx).astype(np.float32)
    S = kf.shape[-2]; g = kf.reshape(kf.shape[:-2] + (S // pool, pool, kf.shape[-1]))
    n = min(pool, 4)
    return OD._orig["f32_to_e4m3"](g[..., :n, :].sum(axis=-2, dtype=np.float32) * np.float32(1.0 / n))


def _expand_no_mask(block_ids, pos, pool):
    out = np.full(block_ids.shape[0] * pool, -1, np.int32)
    for i, b in enumerate(block_ids):
        if b >= 0:
            out[i * pool:(i + 1) * pool] = [pool * int(b) + r for r in range(pool)]
    return out


def _encode_ties_away(x):
    # round half away from zero instead of half to even: move every exact tie to the code
    # above it in magnitude
    x = np.asarray(x, np.float32)
    codes = OD._orig["f32_to_e4m3"](x)
    v = OD._orig["e4m3_to_f64"](codes)
    a = np.abs(x.astype(np.float64))
    up = (codes & 0x7F) + 1
    nxt = OD._orig["e4m3_to_f64"](np.minimum(up, 0x7E).astype(np.uint8))
    tie_down = (np.abs(v) < a) & np.isclose(a - np.abs(v), nxt - a, rtol=0, atol=0) & ((codes & 0x7F) < 0x7E)
    return np.where(tie_down, (codes & 0x80) | up, codes).astype(np.uint8)


def _pool_max(k_idx, pool=4):
    kf = OD._orig["e4m3_to_f64"](k_idx).astype(np.float32)
    S = kf.shape[-2]; g = kf.reshape(kf.shape[:-2] + (S // 4, 4, kf.shape[-1]))
    return OD._orig["f32_to_e4m3"](g.max(axis=-2))


def _select_pool_last_block_dropped(q_idx_t, w_t, k_dec, pos, k, pool=1, k_pool_dec=None):
    if pool == 1:
        return OD._orig["select_row"](q_idx_t, w_t, k_dec, pos, k, pool, k_pool_dec)
    sc = OD.index_scores_row(q_idx_t, w_t, k_pool_dec, pos, pool=pool)
    blocks = OD.topk_row(sc, min(k_pool_dec.shape[0], pos // pool), k)        # off by one block
    return OD.expand_blocks(blocks, pos, pool), sc


def _attn_no_max_subtraction(q_t, K, V, idx_row, sm_scale):
    sel = np.asarray([i for i in idx_row if i >= 0], dtype=np.int64)
    if sel.size == 0:
        return np.zeros((q_t.shape[0], V.shape[1])), np.full(q_t.shape[0], -np.inf)
    with np.errstate(over="ignore", invalid="ignore"):
        p = np.exp((q_t @ K[sel].T) * sm_scale)
        d = p.sum(axis=1, keepdims=True)
        return (p @ V[sel]) / d, np.log(d)[:, 0]


def _group_first_layer_query(q_idx_t, w_t, k_dec, pos, k, layers, sm_scale, pool=1, k_pool_dec=None):
    idx, _ = OD.select_row(q_idx_t, w_t, k_dec, pos, k, pool, k_pool_dec)
    return idx, [OD.sparse_attn_row(layers[0]["q"], L["K"], L["V"], idx, sm_scale) for L in layers]


def _per_layer_first_layer_indexer(indexer_inputs, pos, k, layers, sm_scale):
    return OD._orig["per_layer_forward_row"]([indexer_inputs[0]] * len(layers), pos, k, layers, sm_scale)


def _set_ok_no_missed_rule(gpu_idx, scores_ref, n_valid, k, pos, rel_band=1e-3, pool=1):
    sel = np.asarray([i for i in gpu_idx if i >= 0], dtype=np.int64)
    keff = min(k, n_valid)
    if sel.size != keff or np.unique(sel).size != sel.size or (sel.size and sel.max() >= n_valid):
        return False, "shape"
    if keff == n_valid:
        return True, "all"
    s = np.asarray(scores_ref[:n_valid], dtype=np.float64)
    tau = np.sort(s)[::-1][keff - 1]
    return (not (s[sel] < tau - rel_band * abs(tau)).any()), "below only"


def _set_ok_no_count_rule(gpu_idx, scores_ref, n_valid, k, pos, rel_band=1e-3, pool=1):
    sel = np.asarray([i for i in gpu_idx if i >= 0], dtype=np.int64)
    keff = min(k, n_valid)
    if np.unique(sel).size != sel.size or (sel.size and sel.max() >= n_valid):
        return False, "dup/range"
    s = np.asarray(scores_ref[:n_valid], dtype=np.float64)
    tau = np.sort(s)[::-1][keff - 1]
    band = rel_band * abs(tau)
    if not np.isin(np.nonzero(s > tau + band)[0], sel).all():
        return False, "missed"
    return (not (s[sel] < tau - band).any()), "no count"


def _score_close_abs(gpu, ref, dense_mag, rel=1e-3, floor_rel=1e-5):
    d = np.abs(np.asarray(gpu, np.float64) - np.asarray(ref, np.float64))
    return d <= rel, 0


def _magnitude_signed_w(q_t, w_t, k, pos, pool=1):
    S = k.shape[0]; n = min(S, pos // pool + 1); out = np.zeros(S)
    out[:n] = np.maximum(k[:n] @ q_t.T, 0.0) @ np.asarray(w_t, np.float64)
    return out


MUTANTS = [
    ("index_scores_row", _scores_no_relu, ["test_indexer_single_head_unit_weight_is_relu_dot", "test_indexer_hand_worked_example"]),
    ("index_scores_row", _scores_excl_self, ["test_indexer_causal_rule_includes_self", "test_indexer_brute_force_tiny"]),
    ("index_scores_row", _scores_weights_reversed, ["test_indexer_brute_force_tiny", "test_indexer_hand_worked_example"]),
    ("index_scores_row", _scores_abs_instead_of_relu, ["test_indexer_single_head_unit_weight_is_relu_dot"]),
    ("topk_row", _topk_ties_high_index, ["test_topk_brute_force_sort"]),
    ("topk_row", _topk_smallest, ["test_topk_brute_force_sort", "test_indexer_hand_worked_example"]),
    ("sparse_attn_row", _attn_no_scale, ["test_attention_dense_when_all_keys_selected_matches_torch_sdpa", "test_attention_brute_force_and_permutation"]),
    ("sparse_attn_row", _attn_k_as_v, ["test_attention_dense_when_all_keys_selected_matches_torch_sdpa"]),
    ("sparse_attn_row", _attn_drop_last, ["test_attention_zero_query_is_mean_of_v_and_duplicates_count", "test_attention_brute_force_and_permutation"]),
    ("e4m3_to_f64", _decode_bias8, ["test_e4m3_decode_all_codes_match_torch", "test_e4m3_decode_format_values"]),
    ("f32_to_e4m3", _encode_truncate, ["test_e4m3_encode_matches_torch_in_range"]),
    ("index_pool", _pool_half, ["test_pool_brute_force_and_library_requantisation"]),
    ("expand_blocks", _expand_no_mask, ["test_pool_validity_and_expansion",
                                        "test_select_row_pool_last_block_visible_from_its_first_token"]),
    ("index_pool", _pool_max, ["test_pool_mean_is_exact_then_one_rounding", "test_pool_brute_force_and_library_requantisation",
                               "test_pool_hand_worked_example"]),
    ("index_pool", _pool_half, ["test_pool_hand_worked_example"]),
    ("f32_to_e4m3", _encode_ties_away, ["test_e4m3_encode_matches_torch_in_range", "test_pool_hand_worked_example"]),
    ("select_row", _select_pool_last_block_dropped, ["test_select_row_pool_last_block_visible_from_its_first_token"]),
    ("sparse_attn_row", _attn_no_max_subtraction, ["test_attention_huge_logits_pick_the_argmax_key"]),
    ("sparse_attn_row", _attn_no_scale, ["test_attention_hand_worked_example"]),
    ("sparse_attn_row", _attn_drop_last, ["test_attention_hand_worked_example"]),
    ("sparse_attn_row", _attn_k_as_v, ["test_attention_hand_worked_example"]),
    ("sparse_attn_row", _attn_dedup, ["test_attention_hand_worked_example",
                                      "test_attention_zero_query_is_mean_of_v_and_duplicates_count"]),
    ("group_forward_row", _group_first_layer_query, ["test_indexshare_group_reuses_one_selection"]),
    ("per_layer_forward_row", _per_layer_first_layer_indexer, ["test_per_layer_comparator_selects_with_each_layers_own_indexer"]),
    ("topk_set_ok", _set_ok_no_missed_rule, ["test_topk_acceptance_rule"]),
    ("topk_set_ok", _set_ok_no_count_rule, ["test_topk_acceptance_rule"]),
    ("score_close", _score_close_abs, ["test_score_tolerance_rule_closed_form"]),
    ("score_magnitude_row", _magnitude_signed_w, ["test_score_magnitude_closed_form"]),
    ("index_pool", _pool_fixed_quarter, [("test_pool_factors_2_and_8_identity_brute_force_and_exact_mean", 2),
                                         ("test_pool_factors_2_and_8_identity_brute_force_and_exact_mean", 8)]),
    ("index_pool", _pool_first_four_only, [("test_pool_factors_2_and_8_identity_brute_force_and_exact_mean", 8)]),
    ("expand_blocks", _expand_no_mask, [("test_pool_factor_validity_and_expansion", 2),
                                        ("test_pool_factor_validity_and_expansion", 8)]),
]

if not hasattr(OD, "_orig"):
    OD._orig = {n: getattr(OD, n) for n in
                ["index_scores_row", "topk_row", "sparse_attn_row", "e4m3_to_f64", "f32_to_e4m3",
                 "index_pool", "expand_blocks", "select_row", "group_forward_row", "per_layer_forward_row",
                 "topk_set_ok", "score_close", "score_magnitude_row"]}


@pytest.mark.parametrize("fn,mutant,pins", MUTANTS, ids=[m[1].__name__ for m in MUTANTS])
def test_pins_catch_planted_mistake(monkeypatch, fn, mutant, pins):
    monkeypatch.setattr(OD, fn, mutant)
    monkeypatch.setattr(O, fn, mutant)
    for pin in pins:
        name, args = (pin[0], pin[1:]) if isinstance(pin, tuple) else (pin, ())
        with pytest.raises(AssertionError):
            getattr(P, name)(*args)
