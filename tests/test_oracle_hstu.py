"""Pins for the oracle's HSTU-style masked attention (contextual, candidate
and sliding-window masks; cry-daniel/recsys README, HSTU attention mask
logic).  Each pin reduces a mask feature to something fixed independently of
the oracle's mask code: a library attention call (torch SDPA) on the keys the
reading makes visible, a closed form, or an invariant.  CPU only."""
import numpy as np
import pytest
import torch

from oracle import ptl_oracle as O


def _qkv(rng, T, H=2, Dh=64):
    return [rng.standard_normal((T, H, Dh)) for _ in range(3)]


def _sdpa(q, k, v, causal):
    """torch SDPA (fp64) over [L, H, Dh] arrays."""
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(a)).permute(1, 0, 2)[None] for a in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal)
    return o[0].permute(1, 0, 2).numpy()


def _row_over_keys(q, k, v, i, keys):
    """Query row i attending to exactly the key positions `keys` (SDPA)."""
    keys = np.asarray(keys)
    return _sdpa(q[i:i + 1], k[keys], v[keys], causal=False)[0]


def test_defaults_are_the_causal_attention():
    rng = np.random.default_rng(1)
    cu = [0, 7, 7, 40, 41, 170]
    q, k, v = _qkv(rng, 170)
    np.testing.assert_allclose(O.jagged_hstu_attention(q, k, v, cu),
                               O.jagged_causal_attention(q, k, v, cu), rtol=0, atol=1e-12)


def test_no_mask_is_full_attention_and_permutation_equivariant():
    rng = np.random.default_rng(2)
    cu = [0, 9, 30]
    q, k, v = _qkv(rng, 30)
    out = O.jagged_hstu_attention(q, k, v, cu, causal=False)
    for s, e in ((0, 9), (9, 30)):
        np.testing.assert_allclose(out[s:e], _sdpa(q[s:e], k[s:e], v[s:e], False), atol=1e-12)
    # permuting tokens inside a user permutes its rows (a causal mask would not)
    perm = np.r_[np.arange(9), 9 + rng.permutation(21)]
    out_p = O.jagged_hstu_attention(q[perm], k[perm], v[perm], cu, causal=False)
    np.testing.assert_allclose(out_p, out[perm], atol=1e-12)


def test_context_rows_are_bidirectional_over_the_context_only():
    rng = np.random.default_rng(3)
    L, C = 23, 6
    q, k, v = _qkv(rng, L)
    out = O.jagged_hstu_attention(q, k, v, [0, L], num_contexts=[C])
    np.testing.assert_allclose(out[:C], _sdpa(q[:C], k[:C], v[:C], False), atol=1e-12)
    # history rows are plain causal rows (the contexts precede them)
    np.testing.assert_allclose(out[C:], _sdpa(q, k, v, True)[C:], atol=1e-12)
    # the whole user as context: full attention
    np.testing.assert_allclose(O.jagged_hstu_attention(q, k, v, [0, L], num_contexts=[L]),
                               _sdpa(q, k, v, False), atol=1e-12)


def test_window_one_gives_own_v_and_wide_window_is_causal():
    rng = np.random.default_rng(4)
    cu = [0, 5, 31]
    q, k, v = _qkv(rng, 31)
    np.testing.assert_allclose(O.jagged_hstu_attention(q, k, v, cu, window=1), v, rtol=0, atol=1e-15)
    np.testing.assert_allclose(O.jagged_hstu_attention(q, k, v, cu, window=26),
                               O.jagged_causal_attention(q, k, v, cu), atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_window_rows_see_their_neighbourhood(causal):
    rng = np.random.default_rng(5)
    L, W = 40, 7
    q, k, v = _qkv(rng, L)
    out = O.jagged_hstu_attention(q, k, v, [0, L], causal=causal, window=W)
    for i in (0, 3, 6, 7, 20, 39):
        hi = i if causal else min(L - 1, i + W - 1)
        keys = np.arange(max(0, i - W + 1), hi + 1)
        np.testing.assert_allclose(out[i], _row_over_keys(q, k, v, i, keys), atol=1e-12)


def test_single_candidates_see_history_and_themselves():
    rng = np.random.default_rng(6)
    L, N = 30, 5
    Hs = L - N
    q, k, v = _qkv(rng, L)
    out = O.jagged_hstu_attention(q, k, v, [0, L], num_targets=[N], target_group_size=1)
    # history rows: causal attention of the history alone (no candidate leaks back)
    np.testing.assert_allclose(out[:Hs], _sdpa(q[:Hs], k[:Hs], v[:Hs], True), atol=1e-12)
    for i in range(Hs, L):
        keys = np.r_[np.arange(Hs), i]
        np.testing.assert_allclose(out[i], _row_over_keys(q, k, v, i, keys), atol=1e-12)


def test_candidate_groups():
    rng = np.random.default_rng(7)
    L, N, G = 40, 11, 4  # groups of 4, 4, 3 candidates
    Hs = L - N
    q, k, v = _qkv(rng, L)
    out = O.jagged_hstu_attention(q, k, v, [0, L], num_targets=[N], target_group_size=G)
    for i in range(Hs, L):
        g0 = Hs + (i - Hs) // G * G
        keys = np.r_[np.arange(Hs), np.arange(g0, i + 1)]
        np.testing.assert_allclose(out[i], _row_over_keys(q, k, v, i, keys), atol=1e-12)
    # one group holding every candidate: plain causal attention
    np.testing.assert_allclose(
        O.jagged_hstu_attention(q, k, v, [0, L], num_targets=[N], target_group_size=N),
        _sdpa(q, k, v, True), atol=1e-12)


def test_context_and_candidates_together_per_user():
    rng = np.random.default_rng(8)
    cu = [0, 12, 12, 50]
    q, k, v = _qkv(rng, 50)
    out = O.jagged_hstu_attention(q, k, v, cu, num_contexts=[3, 0, 5], num_targets=[4, 0, 6],
                                  target_group_size=2)
    # user 0: L = 12, C = 3, candidates 8..11 in groups {8, 9}, {10, 11}
    np.testing.assert_allclose(out[0:3], _sdpa(q[0:3], k[0:3], v[0:3], False), atol=1e-12)
    np.testing.assert_allclose(out[3:8], _sdpa(q[0:8], k[0:8], v[0:8], True)[3:8], atol=1e-12)
    np.testing.assert_allclose(out[11], _row_over_keys(q, k, v, 11, np.r_[np.arange(8), 10, 11]),
                               atol=1e-12)
    # user 2 (tokens 12..49) is not affected by user 0's settings
    ref2 = O.jagged_hstu_attention(q[12:], k[12:], v[12:], [0, 38], num_contexts=[5], num_targets=[6],
                                   target_group_size=2)
    np.testing.assert_allclose(out[12:], ref2, atol=1e-12)


def test_every_row_sees_itself_and_masks_are_consistent():
    for L in (1, 2, 9, 33):
        for causal in (True, False):
            for C in (0, 1, L // 2):
                for N in (0, 1, (L - C) // 2):
                    for G in (1, 3):
                        for W in (0, 1, 4):
                            m = O.hstu_user_mask(L, causal, C, N, G, W)
                            assert m.diagonal().all()
                            if causal and C == 0:
                                assert not np.triu(m, 1).any()


def test_out_of_range_counts_are_rejected():
    rng = np.random.default_rng(9)
    q, k, v = _qkv(rng, 10)
    with pytest.raises(ValueError):
        O.jagged_hstu_attention(q, k, v, [0, 10], num_contexts=[6], num_targets=[5])
