"""Pins for the oracle's RepEncoder front end (cti2026 README, RepEncoder
section): the bags against torch's embedding_bag (mode "sum") slot by slot,
closed forms for empty, single and repeated ids, and the LayerNorm + Linear
against torch's LayerNorm over the 14336 values and torch's Linear.  CPU only."""
import numpy as np
import torch

from oracle import ptl_oracle as O
from packed_sequence_transformer_b200 import synthetic as S


def _case(T=6, seed=3, **kw):
    return S.make_rep_case("pin", T, vocab=40, seed=seed, dtype="fp32", **kw)


def test_bags_match_torch_embedding_bag_per_slot():
    c = _case(T=9, max_bag=5)
    bags = O.embedding_bags(c.tables, c.ids, c.bag_offsets, c.num_tokens)
    off = c.bag_offsets
    for s in range(S.REP_SLOTS):
        idx = [c.ids[off[t * 28 + s]:off[t * 28 + s + 1]] for t in range(c.num_tokens)]
        flat = torch.from_numpy(np.concatenate(idx).astype(np.int64))
        starts = torch.from_numpy(np.cumsum([0] + [len(i) for i in idx[:-1]]).astype(np.int64))
        ref = torch.nn.functional.embedding_bag(flat, torch.from_numpy(c.tables[s]).double(), starts,
                                                mode="sum")
        np.testing.assert_allclose(bags[:, s * 512:(s + 1) * 512], ref.numpy(), rtol=0, atol=1e-12)


def test_empty_single_and_repeated_ids():
    c = _case(T=2)
    tables = c.tables
    # token 0: slot 0 empty, slot 1 one id, slot 2 the same id three times;
    # token 1: every slot empty
    ids, sizes = [], []
    for t in range(2):
        for s in range(28):
            if t == 0 and s == 1:
                ids += [5]
            elif t == 0 and s == 2:
                ids += [7, 7, 7]
            sizes.append(len(ids))
    off = np.r_[0, sizes].astype(np.int64)
    bags = O.embedding_bags(tables, np.array(ids, np.int64), off, 2)
    assert not bags[0, :512].any() and not bags[1].any()
    np.testing.assert_array_equal(bags[0, 512:1024], tables[1][5])
    np.testing.assert_allclose(bags[0, 1024:1536], 3 * tables[2][7].astype(np.float64), rtol=0, atol=1e-12)


def test_front_end_is_torch_layer_norm_and_linear():
    c = _case(T=7, random_affine=True)
    out = O.rep_encoder(c.tables, c.ids, c.bag_offsets, c.num_tokens, c.ln_g, c.ln_b, c.w, c.b)
    bags = torch.from_numpy(O.embedding_bags(c.tables, c.ids, c.bag_offsets, c.num_tokens))
    ln = torch.nn.functional.layer_norm(bags, (14336,), torch.from_numpy(c.ln_g).double(),
                                        torch.from_numpy(c.ln_b).double(), eps=1e-5)
    ref = torch.nn.functional.linear(ln, torch.from_numpy(c.w).double(), torch.from_numpy(c.b).double())
    np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-10)


def test_ids_order_inside_a_bag_does_not_matter():
    c = _case(T=4, max_bag=6)
    ids = c.ids.copy()
    off = c.bag_offsets
    rng = np.random.default_rng(0)
    for b in range(len(off) - 1):
        ids[off[b]:off[b + 1]] = rng.permutation(ids[off[b]:off[b + 1]])
    a = O.embedding_bags(c.tables, c.ids, off, c.num_tokens)
    p = O.embedding_bags(c.tables, ids, off, c.num_tokens)
    np.testing.assert_allclose(a, p, rtol=0, atol=1e-12)
