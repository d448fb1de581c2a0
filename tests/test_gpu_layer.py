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
from tests.gpu_util import (assert_close, check_perm_is_stable_sort, dev, host, max_abs,
                            poisoned_workspace, rel_l2, subset_users, tdt)

pytestmark = pytest.mark.gpu

# Acceptance bars: bf16 storage with fp32 accumulation -> max-abs 3e-2 and
# relative L2 1e-2 per layer output; fp32 build -> 1e-4.
LAYER_BF16 = (3e-2, 1e-2)
LAYER_F32 = (1e-4, 1e-5)
# An L-layer stack in bf16 rounds the residual stream twice per layer; for
# |h| up to ~6 one rounding is <= 2^-9 * 8 = 0.016, so the final hidden state
# is held to relative L2 1e-2 and a max-abs of 0.1; the head probabilities to
# 5e-3.
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


def check_routing(dbg, it, T):
    g_idx = dbg["topk_idx"].cpu().numpy()
    sep = it["gap"] > 1e-3
    assert np.array_equal(g_idx[sep], it["idx"][sep]), \
        f"top-2 differs on {int(np.sum(np.any(g_idx[sep] != it['idx'][sep], 1)))} separated tokens"
    g_perm = dbg["perm"].cpu().numpy()
    g_off = dbg["expert_off"].cpu().numpy()
    if np.array_equal(g_idx, it["idx"]):
        assert np.array_equal(g_perm, it["perm"]) and np.array_equal(g_off, it["off"])
    else:  # near-ties decided the other way: the order must still be the stable sort
        check_perm_is_stable_sort(g_idx, g_perm, g_off)
    return float(np.mean(sep))


def test_config0_fp32_layer():
    c = S.config0()
    out, dbg = run_layer(c)
    ref, it = O.layer_forward(c.x, c.cu_seqlens, c.layers[0], return_intermediates=True)
    assert_close(host(out), ref, *LAYER_F32, what="config0 fp32")
    check_routing(dbg, it, c.total_tokens)


def test_config0_shapes_in_bf16():
    c = S.make_case("c0bf16", lengths=[3, 7, 12, 20], seed=0, dtype="bf16")
    out, dbg = run_layer(c)
    ref, it = O.layer_forward(c.x, c.cu_seqlens, c.layers[0], return_intermediates=True)
    assert_close(host(out), ref, *LAYER_BF16, what="config0 bf16")
    check_routing(dbg, it, c.total_tokens)


def test_config1_bf16_layer():
    c = S.config1()
    out, dbg = run_layer(c)
    ref, it = O.layer_forward(c.x, c.cu_seqlens, c.layers[0], return_intermediates=True)
    assert_close(host(out), ref, *LAYER_BF16, what="config1")
    frac = check_routing(dbg, it, c.total_tokens)
    assert frac > 0.9


def test_config1_random_biases():
    c = S.make_case("c1bias", lengths=S.config1_lengths(), seed=11, dtype="bf16", gate_std=0.1,
                    random_bias=True)
    out, dbg = run_layer(c)
    ref, it = O.layer_forward(c.x, c.cu_seqlens, c.layers[0], return_intermediates=True)
    assert_close(host(out), ref, *LAYER_BF16, what="config1 biases")
    check_routing(dbg, it, c.total_tokens)


def test_config4_skewed_gate_subset():
    c = S.config4()
    out, dbg = run_layer(c)
    g_idx = dbg["topk_idx"].cpu().numpy()
    assert np.mean(g_idx[:, 0] == 0) > 0.98          # the +2 bias wins slot 0
    users = [0, 15]
    rows, cu = subset_users(c, users)
    ref, it = O.layer_forward(c.x[rows], cu, c.layers[0], return_intermediates=True)
    assert_close(host(out)[rows], ref, *LAYER_BF16, what="config4 users 0,15")
    sep = it["gap"] > 1e-3
    assert np.array_equal(g_idx[rows][sep], it["idx"][sep])
    check_perm_is_stable_sort(g_idx, dbg["perm"].cpu().numpy(), dbg["expert_off"].cpu().numpy())


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
    assert_close(host(out), ref, *(LAYER_BF16 if dt == "bf16" else LAYER_F32), what=name)
    check_routing(dbg, it, c.total_tokens)


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


def test_config2_stack_with_head():
    c = S.config2()
    out, probs, n = _run_stack(c)
    ref_h, ref_p = O.stack_forward(c.x, c.cu_seqlens, c.layers, c.head, c.pred_mask)
    ma, rl = assert_close(host(out), ref_h, *STACK_BF16, what="config2 hidden")
    assert int(n.item()) == ref_p.size
    assert_close(host(probs)[:ref_p.size], ref_p, PROBS_ATOL, 1e-2, what="config2 probs")


def test_config3_stack_subset_of_users():
    c = S.config3()
    out, _, _ = _run_stack(c)
    L = c.lengths
    users = sorted(set([int(np.argmax(L)), int(np.argmin(L))] + list(range(0, 390, 40))))
    rows, cu = subset_users(c, users)
    ref = O.stack_forward(c.x[rows], cu, c.layers)
    assert_close(host(out)[rows], ref, *STACK_BF16, what="config3 subset")


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
