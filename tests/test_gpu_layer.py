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
from tests.gpu_util import (NearTieChooser, assert_close, check_perm_is_stable_sort, dev, host,
                            poisoned_workspace, rel_l2, subset_users, tdt)

pytestmark = pytest.mark.gpu

# Acceptance bars: bf16 storage with fp32 accumulation -> max-abs 3e-2 and
# relative L2 1e-2 per layer output; fp32 build -> 1e-4.
LAYER_BF16 = (3e-2, 1e-2)
LAYER_F32 = (1e-4, 1e-5)
# An L-layer bf16 stack rounds the residual stream twice per layer (<= 2^-9
# |h| each, |h| up to ~8), so after 8 layers the final hidden state is held
# to max-abs 0.1 and relative L2 1e-2; head probabilities to 5e-3.
STACK_BF16 = (1e-1, 1e-2)
PROBS_ATOL = 5e-3
# Top-2 routing.  Where the 2nd and 3rd gate probabilities lie within a
# margin, either expert is a correct choice and the layer output jumps with
# it, so the oracle follows the GPU's branch there (after checking that it is
# such a near-tie) and every other choice must match exactly.  The bar's
# margin, 1e-3, applies to the decision taken in the kernel's precision (the
# oracle's bf16-storage mode: the same bf16 x1 feeds the gate on both sides).
# Against the fp64 oracle, whose x1 is not rounded, bf16 storage itself moves
# the probabilities by up to ~1e-3 at gate std 0.1, so there the margin is 1e-2.
ROUTE_MARGIN = 1e-3
EXACT_MARGIN = 1e-2


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


def check_layer(case, out, dbg, tol, rows=None, sub_cu=None):
    """Routing bar in the kernel's precision, then outputs against the fp64
    oracle following the GPU's branch only at validated near-ties, then the
    route order (unique given the choices)."""
    x = case.x if rows is None else case.x[rows]
    cu = case.cu_seqlens if rows is None else sub_cu
    w = case.layers[0]
    g = host(out) if rows is None else host(out)[rows]
    g_idx = dbg["topk_idx"].cpu().numpy()
    g_idx_r = g_idx if rows is None else g_idx[rows]
    bf16 = case.dtype == "bf16"
    if bf16:
        ch_bf = NearTieChooser([g_idx_r], ROUTE_MARGIN)
        O.layer_forward(x, cu, w, storage="bf16", choose=lambda p, i: ch_bf(0, p, i))
        ch_bf.assert_ok()
    ch = NearTieChooser([g_idx_r], EXACT_MARGIN if bf16 else ROUTE_MARGIN)
    ref, it = O.layer_forward(x, cu, w, return_intermediates=True, choose=lambda p, i: ch(0, p, i))
    ch.assert_ok()
    assert_close(g, ref, *tol, what=case.name)
    g_perm = dbg["perm"].cpu().numpy()
    g_off = dbg["expert_off"].cpu().numpy()
    if rows is None:
        assert np.array_equal(g_idx, it["idx"])
        assert np.array_equal(g_perm, it["perm"]) and np.array_equal(g_off, it["off"])
    else:
        check_perm_is_stable_sort(g_idx, g_perm, g_off)
    return ch.followed[0]


def test_config0_fp32_layer():
    c = S.config0()
    out, dbg = run_layer(c)
    check_layer(c, out, dbg, LAYER_F32)


def test_config0_shapes_in_bf16():
    c = S.make_case("c0bf16", lengths=[3, 7, 12, 20], seed=0, dtype="bf16")
    out, dbg = run_layer(c)
    check_layer(c, out, dbg, LAYER_BF16)


def test_config1_bf16_layer():
    c = S.config1()
    out, dbg = run_layer(c)
    followed = check_layer(c, out, dbg, LAYER_BF16)
    assert followed < 0.01 * c.total_tokens


def test_config1_packing_fp32_layer_at_the_stated_margin():
    """The 60-user / 6823-token packing of the bf16 workload in the fp32
    build, against the plain fp64 oracle (no storage mode in between): top-2
    bit-exact wherever the 2nd-vs-3rd probability gap exceeds 1e-3, the route
    permutation bit-exact, the layer output within 1e-4."""
    c = S.make_case("config1_fp32", num_users=60, total=6823, median=80.0, sigma=1.0, lmax=1024,
                    seed=1, dtype="fp32", gate_std=0.1)
    out, dbg = run_layer(c)
    followed = check_layer(c, out, dbg, LAYER_F32)
    assert followed < 0.001 * c.total_tokens


def test_config1_random_biases():
    c = S.make_case("c1bias", lengths=S.config1_lengths(), seed=11, dtype="bf16", gate_std=0.1,
                    random_bias=True)
    out, dbg = run_layer(c)
    check_layer(c, out, dbg, LAYER_BF16)


def test_config4_skewed_gate_subset():
    c = S.config4()
    out, dbg = run_layer(c)
    g_idx = dbg["topk_idx"].cpu().numpy()
    assert np.mean(np.any(g_idx == 0, axis=1)) > 0.98   # the +2 bias puts expert 0 in the pair
    assert np.mean(g_idx[:, 0] == 0) > 0.9              # ... usually in slot 0
    rows, cu = subset_users(c, [0, 15])
    check_layer(c, out, dbg, LAYER_BF16, rows=rows, sub_cu=cu)


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
    check_layer(c, out, dbg, LAYER_BF16 if dt == "bf16" else LAYER_F32)


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
    chain_out, gidx = _chain_idx(c, sub_rows)
    assert torch.equal(chain_out, out), "stack differs from the chain of single layers"
    # layer 0 sees identical inputs on both sides: the bar's margin; deeper
    # layers see inputs that already differ by each layer's bf16 output rounding
    # (taken after different accumulation orders), so the drift margin applies
    ch_bf = NearTieChooser(gidx, ROUTE_MARGIN, later_margin=EXACT_MARGIN)
    O.stack_forward(x, sub_cu, c.layers, storage="bf16", choose=ch_bf)
    ch_bf.assert_ok()
    ch = NearTieChooser(gidx, EXACT_MARGIN)
    res = O.stack_forward(x, sub_cu, c.layers, c.head, mask, choose=ch)
    ch.assert_ok()
    ref_h = res if c.head is None else res[0]
    g = host(out) if sub_rows is None else host(out)[sub_rows]
    assert_close(g, ref_h, *STACK_BF16, what=c.name)
    if probs is not None:
        ref_p = res[1]
        assert int(n.item()) == ref_p.size
        assert_close(host(probs)[:ref_p.size], ref_p, PROBS_ATOL, 1e-2, what="probs")


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


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_three_layer_stack_equals_chain_and_oracle(dt):
    """Every layer of a stack starts from cleared per-layer routing state:
    the stack equals the chain of single-layer calls bit for bit, and the
    fp32 build stays within its bar of the fp64 oracle after three layers."""
    c = S.make_case("s3", lengths=[3, 7, 12, 20, 130, 257, 1], seed=5, dtype=dt, num_layers=3,
                    gate_std=0.1)
    out, _, _ = _run_stack(c)
    chain_out, gidx = _chain_idx(c)
    assert torch.equal(chain_out, out), "stack differs from the chain of single layers"
    if dt == "fp32":
        ch = NearTieChooser(gidx, EXACT_MARGIN)
        ref = O.stack_forward(c.x, c.cu_seqlens, c.layers, choose=ch)
        ch.assert_ok()
        assert_close(host(out), ref, 3 * LAYER_F32[0], LAYER_F32[1], what=c.name)


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
