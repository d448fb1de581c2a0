"""Pins for the CPU oracle: closed forms, library routines, brute force and
invariants that the pages fix, each chosen so that a plausible slip in the
oracle (a dropped term, a wrong sign or index, a transposed operand, a wrong
mask or scale) fails at least one of them.  CPU only."""
import itertools
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import ptl_oracle as O
from packed_sequence_transformer_b200 import synthetic as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _frac(a):
    return np.array([[float(Fraction(v)) for v in row] for row in a])


def _rand_qkv(rng, T, H=8, Dh=64):
    return [rng.standard_normal((T, H, Dh)) for _ in range(3)]


# ------------------------------------------------------------------ attention
def test_attention_closed_form_golden():
    g = _golden("attention_closed_form.json")
    T = len(g["q0"])
    q = np.zeros((T, 1, g["d_head"]))
    k = np.zeros_like(q)
    v = np.zeros_like(q)
    q[:, 0, 0] = g["q0"]
    k[:, 0, 0] = g["k0"]
    v[:, 0, :3] = np.array(g["v"])
    out = O.jagged_causal_attention(q, k, v, g["cu_seqlens"])
    np.testing.assert_allclose(out[:, 0, :3], _frac(g["expected"]), rtol=0, atol=1e-13)
    assert np.all(out[:, 0, 3:] == 0)


def test_attention_matches_dense_block_causal_mask():
    g = _golden("equivalence_cases.json")["attention"]
    rng = np.random.default_rng(g["seed"])
    q, k, v = _rand_qkv(rng, g["S"], g["H"], g["Dh"])
    a = O.jagged_causal_attention(q, k, v, g["offsets"])
    b = O.dense_masked_attention(q, k, v, g["offsets"])
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_dense_mask_brute_force():
    cu = [0, 2, 2, 5]
    m = O.dense_block_causal_mask(cu)
    user = [0, 0, 2, 2, 2]
    for i in range(5):
        for j in range(5):
            assert m[i, j] == (user[i] == user[j] and j <= i)


def test_attention_single_user_is_torch_causal_sdpa():
    rng = np.random.default_rng(11)
    q, k, v = _rand_qkv(rng, 29)
    out = O.jagged_causal_attention(q, k, v, [0, 29])
    tq, tk, tv = (torch.from_numpy(a).permute(1, 0, 2)[None] for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    np.testing.assert_allclose(out, ref[0].permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)


def test_attention_first_token_outputs_its_own_v():
    rng = np.random.default_rng(12)
    cu = [0, 1, 5, 5, 12, 13]
    q, k, v = _rand_qkv(rng, 13)
    out = O.jagged_causal_attention(q, k, v, cu)
    for s in (0, 1, 5, 12):
        np.testing.assert_allclose(out[s], v[s], rtol=0, atol=1e-15)


def test_attention_equal_keys_give_prefix_mean_of_v():
    rng = np.random.default_rng(13)
    cu = np.array([0, 4, 11, 20])
    T = 20
    q = rng.standard_normal((T, 8, 64))
    v = rng.standard_normal((T, 8, 64))
    k = np.zeros((T, 8, 64))
    for u in range(3):
        k[cu[u]:cu[u + 1]] = rng.standard_normal((1, 8, 64))
    out = O.jagged_causal_attention(q, k, v, cu)
    for u in range(3):
        seg = v[cu[u]:cu[u + 1]]
        n = np.arange(1, len(seg) + 1)[:, None, None]
        np.testing.assert_allclose(out[cu[u]:cu[u + 1]], np.cumsum(seg, axis=0) / n, atol=1e-12)


def test_attention_user_permutation_and_isolation():
    rng = np.random.default_rng(14)
    lengths = [5, 1, 9, 3]
    cu = S.offsets_from_lengths(lengths)
    T = int(cu[-1])
    q, k, v = _rand_qkv(rng, T)
    base = O.jagged_causal_attention(q, k, v, cu)
    order = [2, 0, 3, 1]
    seg = lambda a, u: a[cu[u]:cu[u + 1]]
    q2, k2, v2 = (np.concatenate([seg(a, u) for u in order]) for a in (q, k, v))
    cu2 = S.offsets_from_lengths([lengths[u] for u in order])
    out2 = O.jagged_causal_attention(q2, k2, v2, cu2)
    np.testing.assert_allclose(out2, np.concatenate([seg(base, u) for u in order]), atol=1e-13)
    # empty users anywhere change nothing
    cu3 = S.offsets_from_lengths([0, 5, 0, 1, 9, 0, 0, 3, 0])
    np.testing.assert_allclose(O.jagged_causal_attention(q, k, v, cu3), base, atol=1e-13)
    # a user alone gives the same rows as inside the batch
    alone = O.jagged_causal_attention(seg(q, 2), seg(k, 2), seg(v, 2), [0, 9])
    np.testing.assert_allclose(alone, seg(base, 2), atol=1e-13)


# ------------------------------------------------------------- LN and Linear
def test_layer_norm_is_torch_layer_norm():
    rng = np.random.default_rng(15)
    x = rng.standard_normal((7, 512)) * 3 + 1
    g = rng.standard_normal(512)
    b = rng.standard_normal(512)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (512,), torch.from_numpy(g),
                                         torch.from_numpy(b), eps=1e-5)
    np.testing.assert_allclose(O.layer_norm(x, g, b), ref.numpy(), atol=1e-12)


def test_linear_is_torch_linear():
    rng = np.random.default_rng(16)
    x, W, b = rng.standard_normal((5, 12)), rng.standard_normal((7, 12)), rng.standard_normal(7)
    ref = torch.nn.functional.linear(torch.from_numpy(x), torch.from_numpy(W), torch.from_numpy(b))
    np.testing.assert_allclose(O.linear(x, W, b), ref.numpy(), atol=1e-12)


# ----------------------------------------------------------------------- gate
def test_top2_golden_ties_and_weights():
    g = _golden("moe_route_closed_form.json")["top2"]
    idx, w = O.top2(np.array(g["p"]))
    assert idx.tolist() == g["idx"]
    np.testing.assert_allclose(w, _frac(g["w"]), atol=1e-15)


def test_top2_gaps_golden():
    """top2_gap = p_(2) - p_(3) and top1_gap = p_(1) - p_(2), hand-read off the
    sorted golden rows (a tie inside the pair in row 0, a tie at the pair's
    edge in row 1)."""
    g = _golden("moe_route_closed_form.json")["top2"]
    p = np.array(g["p"])
    np.testing.assert_allclose(O.top2_gap(p), [float(Fraction(v)) for v in g["gap23"]], atol=1e-15)
    np.testing.assert_allclose(O.top1_gap(p), [float(Fraction(v)) for v in g["gap12"]], atol=1e-15)


def test_top2_gaps_are_the_distance_to_another_choice():
    """What the gaps mean for top2 (itself pinned by brute force): raising the
    best left-out expert by less than top2_gap keeps the chosen pair, by more
    changes it; raising the slot-1 expert by less than top1_gap keeps the slot
    order, by more swaps it.  A gap measured between the wrong ranks moves one
    of these thresholds."""
    rng = np.random.default_rng(170)
    p = rng.dirichlet(np.ones(8), size=200)
    idx, _ = O.top2(p)
    g23, g12 = O.top2_gap(p), O.top1_gap(p)
    assert np.all(g23 >= 0) and np.all(g12 >= 0)
    for t in range(p.shape[0]):
        left_out = [e for e in range(8) if e not in idx[t]]
        third = max(left_out, key=lambda e: (p[t, e], -e))
        for frac, same in ((0.99, True), (1.01, False)):
            q = p[t:t + 1].copy()
            q[0, third] += frac * g23[t] + (0.0 if same else 1e-12)
            assert (set(O.top2(q)[0][0]) == set(idx[t])) == same
            q = p[t:t + 1].copy()
            q[0, idx[t, 1]] += frac * g12[t] + (0.0 if same else 1e-12)
            assert (O.top2(q)[0][0, 0] == idx[t, 0]) == same


def test_top2_brute_force_and_weight_invariants():
    rng = np.random.default_rng(17)
    xn2 = rng.standard_normal((64, 512))
    p = O.gate_probs(xn2, rng.standard_normal((8, 512)) * 0.1, rng.standard_normal(8) * 0.1)
    np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-14)
    idx, w = O.top2(p)
    for t in range(64):
        best = max(itertools.permutations(range(8), 2),
                   key=lambda ab: (p[t, ab[0]], p[t, ab[1]], -ab[0], -ab[1]))
        assert tuple(idx[t]) == best
    assert np.all(np.abs(w.sum(-1) - 1) < 1e-15)
    assert np.all(w[:, 0] >= w[:, 1]) and np.all(w[:, 1] >= 0) and np.all(w[:, 0] >= 0.5)


def test_gate_probs_is_torch_softmax_of_logits():
    rng = np.random.default_rng(18)
    xn2, W, b = rng.standard_normal((9, 512)), rng.standard_normal((8, 512)), rng.standard_normal(8)
    ref = torch.softmax(torch.from_numpy(xn2) @ torch.from_numpy(W).T + torch.from_numpy(b), dim=-1)
    np.testing.assert_allclose(O.gate_probs(xn2, W, b), ref.numpy(), atol=1e-14)


def test_gate_large_bias_is_one_hot_choice():
    rng = np.random.default_rng(19)
    xn2 = rng.standard_normal((20, 512))
    b = np.zeros(8)
    b[5], b[2] = 60.0, 50.0
    idx, w = O.top2(O.gate_probs(xn2, rng.standard_normal((8, 512)) * 0.02, b))
    assert np.all(idx[:, 0] == 5) and np.all(idx[:, 1] == 2)


def test_skewed_gate_bias_sends_every_token_to_expert0():
    """Gate bias +2 on expert 0, +1 on expert 1, gate weights N(0, 0.02^2):
    nearly every token picks expert 0 (half of all routes, the most a top-2
    gate can give one expert) and expert 1 is the usual second choice."""
    rng = np.random.default_rng(4)
    xn2 = O.layer_norm(rng.standard_normal((4096, 512)), np.ones(512), np.zeros(512))
    b = np.zeros(8)
    b[0], b[1] = 2.0, 1.0
    idx, _ = O.top2(O.gate_probs(xn2, rng.standard_normal((8, 512)) * 0.02, b))
    cnt, _, _, _ = O.route_build(idx, 8)
    assert cnt[0] / cnt.sum() > 0.49
    assert cnt[1] / cnt.sum() > 0.35


# ---------------------------------------------------------------------- route
def test_route_build_golden():
    g = _golden("moe_route_closed_form.json")["route"]
    cnt, off, perm, pos = O.route_build(np.array(g["idx"]), g["num_experts"])
    assert cnt.tolist() == g["cnt"] and off.tolist() == g["off"]
    assert perm.tolist() == g["perm"] and pos.tolist() == g["pos"]


def test_route_build_brute_force():
    rng = np.random.default_rng(20)
    for T in (1, 2, 7, 33):
        idx = np.stack([rng.choice(8, 2, replace=False) for _ in range(T)])
        cnt, off, perm, pos = O.route_build(idx, 8)
        expect = []
        for e in range(8):
            for r in range(2 * T):
                if idx[r // 2, r % 2] == e:
                    expect.append(r)
        assert perm.tolist() == expect
        assert sorted(perm.tolist()) == list(range(2 * T))
        assert np.all(pos[perm] == np.arange(2 * T))
        for e in range(8):
            assert off[e + 1] - off[e] == np.sum(idx == e) == cnt[e]


# ------------------------------------------------------------------------ MoE
def test_moe_golden():
    g = _golden("moe_route_closed_form.json")["moe"]
    E = 3
    w1 = np.stack([np.eye(2)] * E)
    b1 = np.zeros((E, 2))
    w2 = np.stack([(e + 1) * np.eye(2) for e in range(E)])
    b2 = np.array([[e, 0.0] for e in range(E)])
    out, _, _ = O.moe_routed(np.array(g["x"]), np.array(g["idx"]), np.array(g["w"]), w1, b1, w2, b2)
    np.testing.assert_allclose(out, np.array(g["expected"]), atol=1e-14)


def _rand_moe(rng, T, D=64, F=96, E=8):
    xn2 = rng.standard_normal((T, D))
    w1 = rng.standard_normal((E, F, D)) * 0.1
    b1 = rng.standard_normal((E, F)) * 0.1
    w2 = rng.standard_normal((E, D, F)) * 0.1
    b2 = rng.standard_normal((E, D)) * 0.1
    p = O.gate_probs(xn2, rng.standard_normal((E, D)), rng.standard_normal(E))
    idx, w = O.top2(p)
    return xn2, idx, w, w1, b1, w2, b2


def test_moe_routed_equals_dense_all_experts():
    rng = np.random.default_rng(21)
    args = _rand_moe(rng, 50)
    routed, _, _ = O.moe_routed(*args)
    np.testing.assert_allclose(routed, O.moe_dense_all_experts(*args), atol=1e-12)


def test_moe_identical_experts_reduce_to_one_ffn():
    rng = np.random.default_rng(22)
    xn2, idx, w, w1, b1, w2, b2 = _rand_moe(rng, 30)
    w1[:], b1[:], w2[:], b2[:] = w1[3], b1[3], w2[3], b2[3]
    out, _, _ = O.moe_routed(xn2, idx, w, w1, b1, w2, b2)
    ffn = np.maximum(xn2 @ w1[0].T + b1[0], 0) @ w2[0].T + b2[0]
    np.testing.assert_allclose(out, ffn, atol=1e-12)


def test_moe_route_major_rows():
    """Route r = 2t + k holds expert idx[t, k] applied to token t."""
    rng = np.random.default_rng(23)
    xn2, idx, w, w1, b1, w2, b2 = _rand_moe(rng, 9)
    _, y, _ = O.moe_routed(xn2, idx, w, w1, b1, w2, b2)
    for t in range(9):
        for kk in range(2):
            e = idx[t, kk]
            ref = np.maximum(w1[e] @ xn2[t] + b1[e], 0) @ w2[e].T + b2[e]
            np.testing.assert_allclose(y[2 * t + kk], ref, atol=1e-12)


# ---------------------------------------------------------------------- layer
def _small_case(seed=30, lengths=(3, 1, 6), random_bias=True):
    return S.make_case("pin", lengths=list(lengths), seed=seed, dtype="fp32",
                       random_bias=random_bias, num_layers=2, with_head=True)


def test_layer_zero_weights_is_identity():
    c = _small_case()
    w = {k: np.zeros_like(v) for k, v in c.layers[0].items()}
    w["ln1_g"][:] = 1
    w["ln2_g"][:] = 1
    np.testing.assert_array_equal(O.layer_forward(c.x, c.cu_seqlens, w), c.x)


def test_layer_zero_query_weights_give_prefix_mean_of_v():
    """With the Q block of Wqkv (rows 0..511) and its bias zero every score
    is 0, so each token's attention output is the mean of V over its user's
    prefix; V must be the third 512-row block of Wqkv."""
    c = _small_case()
    w = dict(c.layers[0])
    w["w_qkv"] = w["w_qkv"].copy()
    w["w_qkv"][:512] = 0
    w["b_qkv"] = w["b_qkv"].copy()
    w["b_qkv"][:512] = 0
    _, it = O.layer_forward(c.x, c.cu_seqlens, w, return_intermediates=True)
    xn = torch.nn.functional.layer_norm(torch.from_numpy(c.x.astype(np.float64)), (512,),
                                        eps=1e-5).numpy()
    V = xn @ w["w_qkv"][1024:].astype(np.float64).T + w["b_qkv"][1024:]
    cu = c.cu_seqlens
    expect = np.zeros_like(V)
    for u in range(len(cu) - 1):
        seg = V[cu[u]:cu[u + 1]]
        expect[cu[u]:cu[u + 1]] = np.cumsum(seg, 0) / np.arange(1, len(seg) + 1)[:, None]
    np.testing.assert_allclose(it["attn"], expect, atol=1e-12)
    np.testing.assert_allclose(it["x1"], c.x + expect @ w["w_o"].astype(np.float64).T + w["b_o"],
                               atol=1e-12)


def test_layer_constant_expert_output_adds_constant():
    """W2 = 0 and b2[e] = c for every expert: the MoE adds exactly c (the
    renormalised weights sum to one)."""
    c = _small_case()
    w = dict(c.layers[0])
    w["w2"] = np.zeros_like(w["w2"])
    cvec = np.linspace(-1, 1, 512)
    w["b2"] = np.tile(cvec, (8, 1))
    out, it = O.layer_forward(c.x, c.cu_seqlens, w, return_intermediates=True)
    np.testing.assert_allclose(out, it["x1"] + cvec, atol=1e-12)


def test_stack_is_composition_and_head_pins():
    c = _small_case()
    h1 = O.layer_forward(c.x, c.cu_seqlens, c.layers[0])
    h2 = O.layer_forward(h1, c.cu_seqlens, c.layers[1])
    hs, probs = O.stack_forward(c.x, c.cu_seqlens, c.layers, c.head, c.pred_mask)
    np.testing.assert_array_equal(hs, h2)
    assert probs.shape == (int(c.pred_mask.sum()),)
    full = O.head_forward(hs, c.head)
    np.testing.assert_array_equal(probs, full[c.pred_mask.astype(bool)])


def test_head_clamp_and_sigmoid_values():
    x = np.tile(np.array([1.0, -1.0]), (3, 256))
    ones, zeros = np.ones(512), np.zeros(512)
    big = {"lnf_g": ones, "lnf_b": zeros, "w": 100 * x[0], "b": np.zeros(1)}
    assert np.allclose(O.head_forward(x, big), 0.9999996940977731, rtol=0, atol=1e-15)
    neg = {"lnf_g": ones, "lnf_b": zeros, "w": -100 * x[0], "b": np.zeros(1)}
    assert np.allclose(O.head_forward(x, neg), 3.059022269256247e-07, rtol=1e-12, atol=0)
    half = {"lnf_g": ones, "lnf_b": zeros, "w": zeros, "b": np.array([0.5])}
    assert np.allclose(O.head_forward(x, half), 0.6224593312018546, rtol=0, atol=1e-15)
    mask = np.array([0, 1, 1], np.uint8)
    assert O.head_forward(x, half, mask).shape == (2,)


def test_head_final_layer_norm_applies():
    """The head normalises first: scaling a row leaves its probability unchanged."""
    rng = np.random.default_rng(31)
    x = rng.standard_normal((4, 512))
    hd = {"lnf_g": np.ones(512), "lnf_b": np.zeros(512), "w": rng.standard_normal(512) * 0.05,
          "b": np.array([0.1])}
    np.testing.assert_allclose(O.head_forward(x, hd), O.head_forward(3.0 * x + 2.0, hd), atol=1e-6)


# ------------------------------------------------------------ input generator
def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(40)
    a = rng.standard_normal(10000).astype(np.float32) * 10
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(S.round_to_bf16(a), ref)


def test_generated_packings():
    L = S.config1_lengths()
    assert L.sum() == 6823 and len(L) == 60 and L.min() >= 1 and L.max() <= 1024
    c = S.config0()
    assert c.cu_seqlens.tolist() == [0, 3, 10, 22, 42]


# ---------------------------------------------------- bf16 storage precision
def test_round_bf16_matches_torch_conversion():
    rng = np.random.default_rng(41)
    a = np.concatenate([rng.standard_normal(20000) * 7, [0.0, -0.0, 1.0, 1.00390625, 1.01171875,
                                                          65504.0, 1e-30, -3.3e38]])
    ref = torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_bf16(a), ref)
    np.testing.assert_array_equal(O.round_bf16(O.round_bf16(a)), O.round_bf16(a))


def test_bf16_storage_mode_stays_within_bf16_error_of_exact():
    c = S.make_case("st", lengths=[30, 1, 70], seed=42, dtype="bf16", gate_std=0.1, random_bias=True)
    ex, it = O.layer_forward(c.x, c.cu_seqlens, c.layers[0], return_intermediates=True)
    bf, itb = O.layer_forward(c.x, c.cu_seqlens, c.layers[0], return_intermediates=True,
                              storage="bf16")
    same = np.all(it["idx"] == itb["idx"], axis=1)
    assert same.mean() > 0.95
    assert np.max(np.abs(bf[same] - ex[same])) < 3e-2
    assert np.array_equal(bf, O.round_bf16(bf))          # stored output is on the bf16 grid
    assert not np.array_equal(bf, ex)


BF16_STORED = ("xn", "qkv", "attn", "xn2", "hidden", "y", "out")


def _bf16_storage_case():
    c = S.make_case("st_pts", lengths=[9, 1, 20], seed=43, dtype="bf16", gate_std=0.1, random_bias=True)
    return c, O.layer_forward(c.x, c.cu_seqlens, c.layers[0], return_intermediates=True,
                              storage="bf16")


def test_bf16_storage_rounding_points():
    """Reading of bf16 inference with fp32 accumulation (cti2026 README: bf16
    activations, fp32 softmax statistics): every activation the layer stores
    -- LayerNorm1 output, q/k/v, attention output, LayerNorm2 output, expert
    hidden rows, each route's expert output and the layer output -- lies on
    the bf16 grid; the residual x1 = x + attn Wo^T + b_o is kept exact (an
    fp32 buffer, not a bf16 one); the gate reads the LayerNorm2 row before it
    is stored, so p is the softmax of the unrounded LayerNorm2 output."""
    c, (out, it) = _bf16_storage_case()
    w = c.layers[0]
    for name in BF16_STORED:
        a = np.asarray(it[name])
        if name in ("hidden", "y"):
            a = a[np.any(a != 0, axis=1)]
        assert np.array_equal(a, O.round_bf16(a)), f"{name} is stored in bf16"
    x1 = np.asarray(c.x, np.float64) + np.asarray(it["attn"]) @ np.asarray(w["w_o"], np.float64).T
    if w.get("b_o") is not None:
        x1 = x1 + np.asarray(w["b_o"], np.float64)
    np.testing.assert_allclose(it["x1"], x1, rtol=0, atol=1e-12)
    assert not np.array_equal(it["x1"], O.round_bf16(it["x1"]))
    xn2_exact = O.layer_norm(it["x1"], w["ln2_g"], w["ln2_b"])
    p = torch.softmax(torch.from_numpy(xn2_exact @ np.asarray(w["w_gate"], np.float64).T
                                       + np.asarray(w["b_gate"], np.float64)), dim=-1).numpy()
    np.testing.assert_allclose(it["p"], p, rtol=0, atol=1e-14)
