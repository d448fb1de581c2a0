"""Layer and stack parity on the GPU (through the C ABI) against the CPU
oracle on the five seeded workloads, plus edge cases and the device-side
error paths.  Where a workload is too large for the fp64 oracle, a subset of
whole users is checked (users are independent: the oracle pins show a
user's rows do not depend on the other users)."""
import numpy as np
import pytest
import torch

from oracle import ptl_oracle as O
from packed_sequence_transformer_b200 import ptl
from packed_sequence_transformer_b200 import synthetic as S
from tests.gpu_util import (assert_close, check_near_tie_choice, check_perm_is_stable_sort, dev,
                            host, max_abs, poisoned_workspace, rel_l2, routing_flips, subset_users,
                            taint_mask, tdt)

pytestmark = pytest.mark.gpu

# Acceptance bars: bf16 storage with fp32 accumulation -> max-abs 3e-2 and
# relative L2 1e-2 per layer output; fp32 build -> 1e-4.  They apply where
# the result is unique: a token whose 2nd and 3rd gate probabilities sit
# within 1e-3 may legitimately get either expert, and the layer output jumps
# with that choice, so such tokens are checked for validity instead.
LAYER_BF16 = (3e-2, 1e-2)
LAYER_F32 = (1e-4, 1e-5)
# An L-layer bf16 stack rounds the residual stream twice per layer (<= 2^-9
# |h| each, |h| up to ~8), so after 8 layers the final hidden state is held
# to max-abs 0.1 and relative L2 1e-2 on the tokens whose user-causal context
# routed identically at every layer; head probabilities to 5e-3.
STACK_BF16 = (1e-1, 1e-2)
PROBS_ATOL = 5e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    ptl.lib()


def run_layer(case, with_debug=True, ws=None):
    td = tdt(case.dtype)
    T, U = case.total_tokens, case.num_users
    ws = ws if ws is not None else poisoned_workspace(T, U, case.dtype)
    x = dev(case.x, td)
    out = torch.full_like(x, float("nan"))
    dbg = None
    if with_debug:
        dbg = {"topk_idx": torch.full((T, 2), -1, dtype=torch.int32, device="cuda"),
               "topk_w": torch.zeros(T, 2, dtype=torch.float32, device="cuda"),
               "perm": torch.full((2 * T,), -1, dtype=torch.int32, device="cuda"),
               "expert_off": torch.full((9,), -1, dtype=torch.int32, device="cuda")}
    ptl.layer_forward(x, out, dev(case.cu_seqlens, torch.int32),
                      ptl.to_device_layer(case.layers[0], case.dtype), ws, debug=dbg)
    torch.cuda.synchronize()
    assert ptl.last_device_error(ws) == 0
    return out, dbg


def check_layer(case, out, dbg, it, ref, tol, rows=None, wts=None):
    """Layer parity where it is unique + validity where a near-tie allowed a
    different choice + bit-exact route order."""
    g = host(out) if rows is None else host(out)[rows]
    g_idx = dbg["topk_idx"].cpu().numpy()
    g_idx_r = g_idx if rows is None else g_idx[rows]
    setflip, ordflip = routing_flips(g_idx_r, it)
    assert_close(g[~setflip], ref[~setflip], *tol, what=case.name)
    check_near_tie_choice(np.where(setflip)[0], g_idx_r, it, wts or case.layers[0], g[setflip], tol)
    g_perm = dbg["perm"].cpu().numpy()
    g_off = dbg["expert_off"].cpu().numpy()
    if rows is None and not setflip.any() and not ordflip.any():
        assert np.array_equal(g_perm, it["perm"]) and np.array_equal(g_off, it["off"])
    else:  # the order that is unique given the GPU's own choices: a stable sort
        check_perm_is_stable_sort(g_idx, g_perm, g_off)
    return int(setflip.sum()), int(ordflip.sum())


def test_config0_fp32_layer():
    c = S.config0()
    out, dbg = run_layer(c)
    ref, it = O.layer_forward(c.x, c.cu_seqlens, c.layers[0], return_intermediates=True)
    check_layer(c, out, dbg, it, ref, LAYER_F32)


def test_config0_shapes_in_bf16():
    c = S.make_case("c0bf16", lengths=[3, 7, 12, 20], seed=0, dtype="bf16")
    out, dbg = run_layer(c)
    ref, it = O.layer_forward(c.x, c.cu_seqlens, c.layers[0], return_intermediates=True)
    check_layer(c, out, dbg, it, ref, LAYER_BF16)


def test_config1_bf16_layer():
    c = S.config1()
    out, dbg = run_layer(c)
    ref, it = O.layer_forward(c.x, c.cu_seqlens, c.layers[0], return_intermediates=True)
    nset, nord = check_layer(c, out, dbg, it, ref, LAYER_BF16)
    assert nset + nord < 0.01 * c.total_tokens


def test_config1_random_biases():
    c = S.make_case("c1bias", lengths=S.config1_lengths(), seed=11, dtype="bf16", gate_std=0.1,
                    random_bias=True)
    out, dbg = run_layer(c)
    ref, it = O.layer_forward(c.x, c.cu_seqlens, c.layers[0], return_intermediates=True)
    check_layer(c, out, dbg, it, ref, LAYER_BF16)


def test_config4_skewed_gate_subset():
    c = S.config4()
    out, dbg = run_layer(c)
    g_idx = dbg["topk_idx"].cpu().numpy()
    assert np.mean(g_idx[:, 0] == 0) > 0.98          # the +2 bias wins slot 0
    users = [0, 15]
    rows, cu = subset_users(c, users)
    ref, it = O.layer_forward(c.x[rows], cu, c.layers[0], return_intermediates=True)
    check_layer(c, out, dbg, it, ref, LAYER_BF16, rows=rows)


EDGE = {
    "one_token": [1],
    "empty_users_around": [0, 0, 5, 0, 1, 0],
    "tile_boundaries": [127, 128, 129, 255, 256, 257],
    "ragged_many": [3, 1, 40, 0, 77, 130, 2, 9, 300, 1],
}


@pytest.mark.parametrize("name", list(EDGE))
@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_edge_packings(name, dt):
    c = S.make_case(name, lengths=EDGE[name], seed=21, dtype=dt, gate_std=0.1, random_bias=True)
    out, dbg = run_layer(c)
    ref, it = O.layer_forward(c.x, c.cu_seqlens, c.layers[0], return_intermediates=True)
    check_layer(c, out, dbg, it, ref, LAYER_BF16 if dt == "bf16" else LAYER_F32)


def test_empty_users_do_not_change_rows():
    a = S.make_case("a", lengths=[50, 7, 200], seed=5, dtype="bf16", gate_std=0.1)
    b = S.make_case("a", lengths=[50, 7, 200], seed=5, dtype="bf16", gate_std=0.1)
    b.cu_seqlens = S.offsets_from_lengths([0, 50, 0, 0, 7, 200, 0])
    oa, _ = run_layer(a, with_debug=False)
    ob, _ = run_layer(b, with_debug=False)
    assert torch.equal(oa, ob)


def test_deterministic_repeat():
    c = S.config1()
    ws = ptl.alloc_workspace(c.total_tokens, c.num_users, "bf16")
    o1, _ = run_layer(c, with_debug=False, ws=ws)
    o2, _ = run_layer(c, with_debug=False, ws=ws)
    assert torch.equal(o1, o2)


def _run_stack(c, ws=None):
    td = tdt(c.dtype)
    T, U = c.total_tokens, c.num_users
    ws = ws if ws is not None else poisoned_workspace(T, U, c.dtype)
    x = dev(c.x, td)
    out = torch.empty_like(x)
    layers = [ptl.to_device_layer(w, c.dtype) for w in c.layers]
    probs = n = mask = head = None
    if c.head is not None:
        head = ptl.to_device_head(c.head)
        mask = dev(c.pred_mask, torch.uint8)
        probs = torch.full((T,), -1.0, dtype=torch.float32, device="cuda")
        n = torch.zeros(1, dtype=torch.int32, device="cuda")
    ptl.stack_forward(x, out, dev(c.cu_seqlens, torch.int32), layers, ws, head=head, pred_mask=mask,
                      probs=probs, n_pred=n)
    torch.cuda.synchronize()
    assert ptl.last_device_error(ws) == 0
    return out, probs, n


def _chain_idx(c, rows=None):
    """Per-layer top-2 choices of the same computation run as a chain of
    single-layer calls (the chain is checked bit-identical to the stack)."""
    T, U = c.total_tokens, c.num_users
    ws = ptl.alloc_workspace(T, U, c.dtype)
    cu = dev(c.cu_seqlens, torch.int32)
    h = dev(c.x, tdt(c.dtype))
    idx = []
    for w in c.layers:
        out = torch.empty_like(h)
        dbg = {"topk_idx": torch.empty(T, 2, dtype=torch.int32, device="cuda")}
        ptl.layer_forward(h, out, cu, ptl.to_device_layer(w, c.dtype), ws, debug=dbg)
        gi = dbg["topk_idx"].cpu().numpy()
        idx.append(gi if rows is None else gi[rows])
        h = out
    torch.cuda.synchronize()
    return h, idx


def _check_stack(c, out, sub_rows, sub_cu, probs=None, n=None):
    x = c.x if sub_rows is None else c.x[sub_rows]
    mask = c.pred_mask if (c.pred_mask is None or sub_rows is None) else c.pred_mask[sub_rows]
    res = O.stack_forward(x, sub_cu, c.layers, c.head, mask, return_intermediates=True)
    ref_h, per = res[0], res[-1]
    chain_out, gidx = _chain_idx(c, sub_rows)
    assert torch.equal(chain_out, out), "stack differs from the chain of single layers"
    flips = np.zeros(len(ref_h), bool)
    for l, it in enumerate(per):
        setflip, _ = routing_flips(gidx[l], it) if l == 0 else (
            np.any(np.sort(gidx[l], 1) != np.sort(it["idx"], 1), axis=1), None)
        flips |= setflip
    taint = taint_mask(sub_cu, flips)
    assert taint.mean() < 0.9, "too few tokens with a unique result to compare"
    g = host(out) if sub_rows is None else host(out)[sub_rows]
    assert_close(g[~taint], ref_h[~taint], *STACK_BF16, what=c.name + " untainted")
    assert rel_l2(g[~flips], ref_h[~flips]) <= 2e-2
    if probs is not None:
        ref_p = res[1]
        assert int(n.item()) == ref_p.size
        keep = ~taint[np.asarray(mask).astype(bool)]
        assert_close(host(probs)[:ref_p.size][keep], ref_p[keep], PROBS_ATOL, 1e-2, what="probs")


def test_config2_stack_with_head():
    c = S.config2()
    out, probs, n = _run_stack(c)
    _check_stack(c, out, None, c.cu_seqlens, probs, n)


def test_config3_stack_subset_of_users():
    c = S.config3()
    out, _, _ = _run_stack(c)
    L = c.lengths
    users = sorted(set([int(np.argmax(L)), int(np.argmin(L))] + list(range(0, 390, 40))))
    rows, cu = subset_users(c, users)
    _check_stack(c, out, rows, cu)


def test_stack_of_one_equals_layer():
    c = S.make_case("s1", lengths=[10, 300, 1], seed=9, dtype="bf16", gate_std=0.1)
    o_layer, _ = run_layer(c, with_debug=False)
    o_stack, _, _ = _run_stack(c)
    assert torch.equal(o_layer, o_stack)


@pytest.mark.parametrize("bad", ["not_monotone", "first_not_zero", "last_not_T"])
def test_bad_offsets_reported(bad):
    c = S.make_case("bad", lengths=[5, 6, 7], seed=3, dtype="bf16")
    cu = c.cu_seqlens.copy()
    if bad == "not_monotone":
        cu[1], cu[2] = cu[2], cu[1]
    elif bad == "first_not_zero":
        cu[0] = 1
    else:
        cu[-1] = cu[-1] - 1
    T = c.total_tokens
    ws = ptl.alloc_workspace(T, 3, "bf16")
    x = dev(c.x, torch.bfloat16)
    out = torch.empty_like(x)
    ptl.layer_forward(x, out, dev(cu, torch.int32), ptl.to_device_layer(c.layers[0], "bf16"), ws)
    assert ptl.last_device_error(ws) == ptl.STATUS_CODE["PTL_ERR_BAD_OFFSETS"]
    # the workspace stays usable: a good call afterwards succeeds
    ptl.layer_forward(x, out, dev(c.cu_seqlens, torch.int32),
                      ptl.to_device_layer(c.layers[0], "bf16"), ws)
    assert ptl.last_device_error(ws) == 0


def test_zero_tokens_is_a_no_op():
    ws = ptl.alloc_workspace(1, 1, "bf16")
    x = torch.empty(0, 512, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(0, 512, dtype=torch.bfloat16, device="cuda")
    cu = torch.zeros(2, dtype=torch.int32, device="cuda")
    c = S.make_case("z", lengths=[1], seed=1, dtype="bf16")
    ptl.layer_forward(x, out, cu, ptl.to_device_layer(c.layers[0], "bf16"), ws)
