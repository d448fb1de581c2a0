"""Plant plausible mistakes in the oracle (on the CPU, by monkeypatching) and
check that at least one pin in test_oracle_pins fails for each.  This shows
the pins constrain every step rather than restating the oracle."""
import numpy as np
import pytest

from oracle import ptl_oracle as O
import tests.test_oracle_pins as P


def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


def test_wrong_softmax_scale_is_caught(monkeypatch):
    orig = O.jagged_causal_attention
    monkeypatch.setattr(O, "jagged_causal_attention",
                        lambda q, k, v, cu, scale=None: orig(q, k, v, cu, scale=1.0 / 64))
    assert _fails(P.test_attention_closed_form_golden)
    assert _fails(P.test_attention_single_user_is_torch_causal_sdpa)


def test_missing_causal_mask_is_caught(monkeypatch):
    def no_causal(q, k, v, cu, scale=None):
        q, k, v = (np.asarray(a, np.float64) for a in (q, k, v))
        out = np.zeros_like(q)
        for u in range(len(cu) - 1):
            s, e = int(cu[u]), int(cu[u + 1])
            if e == s:
                continue
            for h in range(q.shape[1]):
                S = q[s:e, h] @ k[s:e, h].T / 8.0
                out[s:e, h] = O._softmax_rows(S) @ v[s:e, h]
        return out
    monkeypatch.setattr(O, "jagged_causal_attention", no_causal)
    assert _fails(P.test_attention_first_token_outputs_its_own_v)
    assert _fails(P.test_attention_matches_dense_block_causal_mask)


def test_cross_user_leak_is_caught(monkeypatch):
    orig = O.jagged_causal_attention
    monkeypatch.setattr(O, "jagged_causal_attention",
                        lambda q, k, v, cu, scale=None: orig(q, k, v, [0, int(cu[-1])], scale))
    assert _fails(P.test_attention_user_permutation_and_isolation)
    assert _fails(P.test_attention_closed_form_golden)


def test_swapped_k_and_v_blocks_are_caught(monkeypatch):
    orig = O.split_qkv

    def swapped(qkv):
        q, k, v = orig(qkv)
        return q, v, k
    monkeypatch.setattr(O, "split_qkv", swapped)
    assert _fails(P.test_layer_zero_query_weights_give_prefix_mean_of_v)


def test_tie_break_to_higher_index_is_caught(monkeypatch):
    def top2_hi(p):
        p = np.asarray(p, np.float64)
        E = p.shape[1]
        order = E - 1 - np.argsort(-p[:, ::-1], axis=-1, kind="stable")
        idx = order[:, :2]
        pt = np.take_along_axis(p, idx, axis=-1)
        return idx, pt / pt.sum(-1, keepdims=True)
    monkeypatch.setattr(O, "top2", top2_hi)
    assert _fails(P.test_top2_golden_ties_and_weights)


def test_missing_renormalisation_is_caught(monkeypatch):
    def top2_raw(p):
        p = np.asarray(p, np.float64)
        idx = np.argsort(-p, axis=-1, kind="stable")[:, :2]
        return idx, np.take_along_axis(p, idx, axis=-1)
    monkeypatch.setattr(O, "top2", top2_raw)
    assert _fails(P.test_layer_constant_expert_output_adds_constant)
    assert _fails(P.test_top2_golden_ties_and_weights)


def test_unstable_route_order_is_caught(monkeypatch):
    orig = O.route_build

    def unstable(idx, E):
        cnt, off, perm, pos = orig(idx, E)
        perm = perm.copy()
        for e in range(E):
            perm[off[e]:off[e + 1]] = perm[off[e]:off[e + 1]][::-1]
        pos = np.empty_like(perm)
        pos[perm] = np.arange(perm.size)
        return cnt, off, perm, pos
    monkeypatch.setattr(O, "route_build", unstable)
    assert _fails(P.test_route_build_golden)
    assert _fails(P.test_route_build_brute_force)


def test_dropped_expert_bias_is_caught(monkeypatch):
    orig = O.moe_routed

    def no_b2(xn2, idx, w, w1, b1, w2, b2, **kw):
        return orig(xn2, idx, w, w1, b1, w2, np.zeros_like(np.asarray(b2, np.float64)), **kw)
    monkeypatch.setattr(O, "moe_routed", no_b2)
    assert _fails(P.test_moe_golden)
    assert _fails(P.test_layer_constant_expert_output_adds_constant)


def test_missing_logit_clamp_is_caught(monkeypatch):
    monkeypatch.setattr(O, "LOGIT_CLAMP", 1e9)
    assert _fails(P.test_head_clamp_and_sigmoid_values)


# ------------------------------------------------- HSTU-style masks
import tests.test_oracle_hstu as PH  # noqa: E402


def _mask_mutant(monkeypatch, edit):
    orig = O.hstu_user_mask

    def mutant(L, causal=True, num_contexts=0, num_targets=0, target_group_size=1, window=0):
        return edit(orig, L, causal, int(num_contexts), int(num_targets), int(target_group_size),
                    int(window))
    monkeypatch.setattr(O, "hstu_user_mask", mutant)


def test_context_rule_dropped_is_caught(monkeypatch):
    _mask_mutant(monkeypatch, lambda f, L, c, C, N, G, W: f(L, c, 0, N, G, W))
    assert _fails(PH.test_context_rows_are_bidirectional_over_the_context_only)


def test_candidate_groups_off_by_one_is_caught(monkeypatch):
    _mask_mutant(monkeypatch, lambda f, L, c, C, N, G, W: f(L, c, C, N, G + 1, W))
    assert _fails(PH.test_candidate_groups)


def test_candidates_leaking_into_history_is_caught(monkeypatch):
    # candidates visible to every later row, as with a plain causal mask
    _mask_mutant(monkeypatch, lambda f, L, c, C, N, G, W: f(L, c, C, 0, G, W))
    assert _fails(PH.test_single_candidates_see_history_and_themselves)


def test_window_off_by_one_is_caught(monkeypatch):
    _mask_mutant(monkeypatch, lambda f, L, c, C, N, G, W: f(L, c, C, N, G, W + 1 if W > 0 else 0))
    assert _fails(PH.test_window_one_gives_own_v_and_wide_window_is_causal)
    assert _fails(lambda: PH.test_window_rows_see_their_neighbourhood(True))


# ------------------------------------------------- RepEncoder front end
import tests.test_oracle_rep as PR  # noqa: E402


def test_slot_mix_up_is_caught(monkeypatch):
    # each slot's sum written one slot block to the right
    orig = O.embedding_bags
    monkeypatch.setattr(O, "embedding_bags",
                        lambda tables, ids, off, T: np.roll(orig(tables, ids, off, T), 512, axis=1))
    assert _fails(PR.test_bags_match_torch_embedding_bag_per_slot)


def test_layer_norm_per_slot_instead_of_whole_row_is_caught(monkeypatch):
    orig_ln = O.layer_norm

    def per_slot(x, g, b, eps=O.LN_EPS):
        x = np.asarray(x, np.float64)
        if x.shape[-1] != 14336:
            return orig_ln(x, g, b, eps)
        parts = [orig_ln(x[..., s * 512:(s + 1) * 512], np.asarray(g)[s * 512:(s + 1) * 512],
                         np.asarray(b)[s * 512:(s + 1) * 512], eps) for s in range(28)]
        return np.concatenate(parts, axis=-1)
    monkeypatch.setattr(O, "layer_norm", per_slot)
    assert _fails(PR.test_front_end_is_torch_layer_norm_and_linear)


# ------------------------------------------------- FP8 (e4m3) operands
import tests.test_oracle_fp8 as P8  # noqa: E402


def _e4m3_mutant(mant_bits=3, tie_even=True, saturate=True, sub_exp=-9):
    def q(x):
        x = np.asarray(x, np.float64)
        a = np.abs(x)
        with np.errstate(divide="ignore"):
            E = np.floor(np.log2(np.where(a > 0, a, 1.0)))
        quantum = np.where(a >= 2.0 ** -6, 2.0 ** (np.maximum(E, -6) - mant_bits), 2.0 ** sub_exp)
        r = np.round(a / quantum) if tie_even else np.floor(a / quantum + 0.5)
        r = r * quantum
        if saturate:
            r = np.minimum(r, 448.0)
        return np.sign(x) * r
    return q


@pytest.mark.parametrize("kw", [dict(mant_bits=4), dict(tie_even=False), dict(sub_exp=-10)])
def test_e4m3_rounding_slips_are_caught(monkeypatch, kw):
    monkeypatch.setattr(O, "quantize_e4m3", _e4m3_mutant(**kw))
    assert _fails(P8.test_rounding_matches_torch_float8_e4m3fn)


def test_missing_saturation_is_caught(monkeypatch):
    monkeypatch.setattr(O, "quantize_e4m3", _e4m3_mutant(saturate=False))
    assert _fails(P8.test_value_set_and_extremes)


# ------------------------------------------------- top-2 margins
def test_gap_measured_from_the_first_expert_is_caught(monkeypatch):
    """p_(1) - p_(3) in place of p_(2) - p_(3): the margin of the routing bar
    would widen silently."""
    def wrong(p):
        ps = -np.sort(-np.asarray(p, np.float64), axis=-1)
        return ps[:, 0] - ps[:, 2]
    monkeypatch.setattr(O, "top2_gap", wrong)
    assert _fails(P.test_top2_gaps_golden)
    assert _fails(P.test_top2_gaps_are_the_distance_to_another_choice)


def test_slot_gap_measured_to_the_third_is_caught(monkeypatch):
    def wrong(p):
        ps = -np.sort(-np.asarray(p, np.float64), axis=-1)
        return ps[:, 0] - ps[:, 2]
    monkeypatch.setattr(O, "top1_gap", wrong)
    assert _fails(P.test_top2_gaps_golden)
    assert _fails(P.test_top2_gaps_are_the_distance_to_another_choice)


# ------------------------------------------------- bf16 storage points
def _skip_nth_rounding(monkeypatch, n):
    """The bf16 storage mode with its n-th rounding call (in layer order:
    LayerNorm1, qkv, attention, LayerNorm2, then per expert hidden and output,
    then the layer output; -1 = the last) left out."""
    orig = O._storage

    def storage(kind):
        rnd = orig(kind)
        if kind != "bf16":
            return rnd
        calls = []

        def mutant(a):
            calls.append(1)
            if len(calls) == n:
                return O._f64(a)
            return rnd(a)
        return mutant
    monkeypatch.setattr(O, "_storage", storage)


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5])
def test_each_dropped_bf16_rounding_point_is_caught(monkeypatch, n):
    _skip_nth_rounding(monkeypatch, n)
    assert _fails(P.test_bf16_storage_rounding_points)


def test_dropped_expert_output_rounding_is_caught(monkeypatch):
    orig = O.moe_routed

    def no_y_round(xn2, idx, w, w1, b1, w2, b2, hidden_round=None):
        out, y, hidden = orig(xn2, idx, w, w1, b1, w2, b2, hidden_round=None)
        if hidden_round is not None:
            hidden = hidden_round(hidden)
        return out, y, hidden
    monkeypatch.setattr(O, "moe_routed", no_y_round)
    assert _fails(P.test_bf16_storage_rounding_points)


def _patch_bf16_intermediate(monkeypatch, name, fn):
    """The bf16 storage mode with intermediate `name` replaced by fn(it)."""
    orig_layer = O.layer_forward

    def layer(x, cu, wts, return_intermediates=False, storage=None, choose=None):
        out, it = orig_layer(x, cu, wts, True, storage, choose)
        if storage == "bf16":
            it = dict(it)
            it[name] = fn(it)
            out = it["out"]
        return (out, it) if return_intermediates else out
    monkeypatch.setattr(O, "layer_forward", layer)


def test_dropped_layer_output_rounding_is_caught(monkeypatch):
    """The layer output left unrounded (x1 + moe stored in fp64)."""
    _patch_bf16_intermediate(monkeypatch, "out", lambda it: it["x1"] + it["moe"])
    assert _fails(P.test_bf16_storage_rounding_points)


def test_rounded_residual_is_caught(monkeypatch):
    """x1 rounded to bf16 (a bf16 residual buffer) instead of kept exact."""
    _patch_bf16_intermediate(monkeypatch, "x1", lambda it: O.round_bf16(it["x1"]))
    assert _fails(P.test_bf16_storage_rounding_points)


def test_gate_on_the_stored_layernorm2_row_is_caught(monkeypatch):
    """The gate fed the bf16-rounded LayerNorm2 row instead of the row before
    it is stored."""
    def p_rounded(it):
        return O.gate_probs(it["xn2"], W["w_gate"], W["b_gate"])
    W = {}
    orig_case = P._bf16_storage_case

    def case():
        c, res = orig_case()
        W.update(c.layers[0])
        res[1]["p"] = p_rounded(res[1])
        return c, res
    monkeypatch.setattr(P, "_bf16_storage_case", case)
    assert _fails(P.test_bf16_storage_rounding_points)
