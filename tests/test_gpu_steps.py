"""Parity of each step of the layer on the GPU (through the C ABI) against
the CPU oracle on the same seeded inputs.  Sizes span several 128-row tiles
with ragged tails; edge cases include empty users, users of length 1 and
users that straddle tile boundaries."""
import numpy as np
import pytest
import torch

from oracle import ptl_oracle as O
from packed_sequence_transformer_b200 import ptl
from packed_sequence_transformer_b200 import synthetic as S
from tests.gpu_util import (assert_close, check_perm_is_stable_sort, dev, host, poisoned_workspace,
                            random_topk)

pytestmark = pytest.mark.gpu

BF = torch.bfloat16
F32 = torch.float32
# bf16 storage, fp32 accumulation: per-step outputs are O(1) and carry one
# bf16 rounding (<= 2^-9 relative, <= 0.01 at |v| = 5) plus the fp32
# accumulation of bf16 products; the fp32 build differs from the fp64 oracle
# only by fp32 rounding.
ATOL_BF16 = 2e-2
RL2_BF16 = 1e-2
ATOL_F32 = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    ptl.lib()


def _weights(seed, dt, gate_std=0.1):
    c = S.make_case("w", lengths=[1], seed=seed, dtype=dt, random_bias=True, gate_std=gate_std)
    return c.layers[0]


@pytest.mark.parametrize("dt,T", [("bf16", 1), ("bf16", 300), ("bf16", 6823), ("fp32", 300)])
def test_qkv_projection(dt, T):
    rng = np.random.default_rng(100 + T)
    x = S.round_to_bf16(rng.standard_normal((T, 512)).astype(np.float32)) if dt == "bf16" else \
        rng.standard_normal((T, 512)).astype(np.float32)
    w = _weights(101, dt)
    td = BF if dt == "bf16" else F32
    ws = poisoned_workspace(T, 1, dt)
    qkv = torch.empty(T, 1536, dtype=td, device="cuda")
    ptl.qkv_projection(dev(x, td), qkv, ptl.to_device_layer(w, dt), ws)
    torch.cuda.synchronize()
    ref = O.linear(O.layer_norm(x, w["ln1_g"], w["ln1_b"]), w["w_qkv"], w["b_qkv"])
    tol = (ATOL_BF16, RL2_BF16) if dt == "bf16" else (ATOL_F32, 1e-5)
    assert_close(host(qkv), ref, *tol, what=f"qkv {dt} T={T}")


ATTN_LENGTHS = {
    "ragged": [1, 127, 128, 129, 0, 300, 5, 513, 0],
    "single_long": [1100],
    "many_short": [1, 2, 3, 1, 7, 64, 65, 0, 1, 30] * 6,
    "config1": None,
}


@pytest.mark.parametrize("name", list(ATTN_LENGTHS))
@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_attention(name, dt):
    lengths = ATTN_LENGTHS[name]
    if lengths is None:
        if dt == "fp32":
            pytest.skip("fp32 attention is the correctness build; config-1 size covered in bf16")
        lengths = S.config1_lengths()
    cu = S.offsets_from_lengths(lengths)
    T = int(cu[-1])
    rng = np.random.default_rng(7)
    qkv = rng.standard_normal((T, 1536)).astype(np.float32)
    if dt == "bf16":
        qkv = S.round_to_bf16(qkv)
    td = BF if dt == "bf16" else F32
    ws = poisoned_workspace(T, len(lengths), dt)
    out = torch.full((T, 512), float("nan"), dtype=td, device="cuda")
    ptl.attention(dev(qkv, td), out, dev(cu, torch.int32), ws)
    torch.cuda.synchronize()
    assert ptl.last_device_error(ws) == 0
    q, k, v = O.split_qkv(qkv)
    ref = O.jagged_causal_attention(q, k, v, cu).reshape(T, 512)
    tol = (ATOL_BF16, RL2_BF16) if dt == "bf16" else (ATOL_F32, 1e-5)
    assert_close(host(out), ref, *tol, what=f"attention {name} {dt}")


def test_attention_first_token_is_its_v_row():
    """First token of every user outputs its own V row (exactly, up to the
    bf16 store of a value that is already bf16)."""
    lengths = [3, 1, 200, 0, 129]
    cu = S.offsets_from_lengths(lengths)
    T = int(cu[-1])
    qkv = S.round_to_bf16(np.random.default_rng(8).standard_normal((T, 1536)).astype(np.float32))
    ws = ptl.alloc_workspace(T, len(lengths), "bf16")
    out = torch.empty(T, 512, dtype=BF, device="cuda")
    ptl.attention(dev(qkv, BF), out, dev(cu, torch.int32), ws)
    torch.cuda.synchronize()
    o = host(out)
    for u in range(len(lengths)):
        if lengths[u]:
            assert np.array_equal(o[cu[u]], qkv[cu[u], 1024:])


@pytest.mark.parametrize("dt,T", [("bf16", 300), ("bf16", 6823), ("fp32", 300)])
def test_out_projection(dt, T):
    rng = np.random.default_rng(200 + T)
    attn = rng.standard_normal((T, 512)).astype(np.float32)
    x = rng.standard_normal((T, 512)).astype(np.float32)
    if dt == "bf16":
        attn, x = S.round_to_bf16(attn), S.round_to_bf16(x)
    w = _weights(201, dt)
    td = BF if dt == "bf16" else F32
    ws = poisoned_workspace(T, 1, dt)
    x1 = torch.empty(T, 512, dtype=F32, device="cuda")  # the residual stream stays fp32
    ptl.out_projection(dev(attn, td), dev(x, td), x1, ptl.to_device_layer(w, dt), ws)
    torch.cuda.synchronize()
    ref = x + O.linear(attn, w["w_o"], w["b_o"])
    tol = (ATOL_BF16, RL2_BF16) if dt == "bf16" else (ATOL_F32, 1e-5)
    assert_close(host(x1), ref, *tol, what=f"out_proj {dt}")


@pytest.mark.parametrize("dt,T", [("bf16", 1), ("bf16", 1000), ("bf16", 6823), ("fp32", 300)])
def test_gate(dt, T):
    rng = np.random.default_rng(300 + T)
    x1 = rng.standard_normal((T, 512)).astype(np.float32) * 1.3 + 0.2   # fp32 residual
    w = _weights(301, dt)
    td = BF if dt == "bf16" else F32
    ws = poisoned_workspace(T, 1, dt)
    xn2 = torch.empty(T, 512, dtype=td, device="cuda")
    idx = torch.empty(T, 2, dtype=torch.int32, device="cuda")
    wt = torch.empty(T, 2, dtype=F32, device="cuda")
    ptl.gate(dev(x1, F32), xn2, idx, wt, ptl.to_device_layer(w, dt), ws)
    torch.cuda.synchronize()
    xn2_ref = O.layer_norm(x1, w["ln2_g"], w["ln2_b"])
    p = O.gate_probs(xn2_ref, w["w_gate"], w["b_gate"])
    idx_ref, w_ref = O.top2(p)
    gap = O.top2_gap(p)
    tol = (ATOL_BF16, RL2_BF16) if dt == "bf16" else (ATOL_F32, 1e-5)
    assert_close(host(xn2), xn2_ref, *tol, what="xn2")
    g_idx = idx.cpu().numpy()
    sep = gap > 1e-3
    assert np.array_equal(g_idx[sep], idx_ref[sep]), "top-2 experts differ on separated tokens"
    same = np.all(g_idx == idx_ref, axis=1)
    assert_close(host(wt)[same], w_ref[same], 1e-4, 1e-4, what="top-2 weights")
    gw = host(wt)
    assert np.all(np.abs(gw.sum(1) - 1) < 1e-6) and np.all(gw[:, 0] >= gw[:, 1])


ROUTE_CASES = ["uniform", "skewed", "two_experts", "tiny"]


@pytest.mark.parametrize("T", [1, 127, 128, 1000, 6823, 65536])
@pytest.mark.parametrize("kind", ROUTE_CASES)
def test_route_build_bit_exact(T, kind):
    rng = np.random.default_rng(400 + T)
    if kind == "uniform":
        idx, _ = random_topk(rng, T)
    elif kind == "skewed":
        e0 = np.where(rng.random(T) < 0.95, 0, rng.integers(1, 8, T))
        e1 = np.where(e0 == 0, np.where(rng.random(T) < 0.8, 1, rng.integers(2, 8, T)), 0)
        idx = np.stack([e0, e1], 1).astype(np.int32)
    elif kind == "two_experts":
        idx = np.tile(np.array([[6, 3]], np.int32), (T, 1))
        idx[::3] = [3, 6]
    else:
        idx = np.tile(np.array([[7, 0]], np.int32), (T, 1))
    ws = poisoned_workspace(T, 1, "bf16")
    perm = torch.full((2 * T,), -7, dtype=torch.int32, device="cuda")
    off = torch.full((9,), -7, dtype=torch.int32, device="cuda")
    ptl.route_build(dev(idx, torch.int32), perm, off, ws)
    torch.cuda.synchronize()
    assert ptl.last_device_error(ws) == 0
    cnt, off_ref, perm_ref, _ = O.route_build(idx, 8)
    assert np.array_equal(off.cpu().numpy(), off_ref)
    assert np.array_equal(perm.cpu().numpy(), perm_ref)


def test_route_build_rejects_bad_expert_id():
    T = 64
    idx = np.zeros((T, 2), np.int32)
    idx[:, 1] = 1
    idx[5, 0] = 9
    ws = ptl.alloc_workspace(T, 1, "bf16")
    perm = torch.empty(2 * T, dtype=torch.int32, device="cuda")
    ptl.route_build(dev(idx, torch.int32), perm, None, ws)
    assert ptl.last_device_error(ws) == ptl.STATUS_CODE["PTL_ERR_SHAPE"]


@pytest.mark.parametrize("dt,T,kind", [("bf16", 300, "uniform"), ("bf16", 6823, "uniform"),
                                       ("bf16", 4000, "skewed"), ("bf16", 1, "uniform"),
                                       ("fp32", 300, "uniform")])
def test_moe(dt, T, kind):
    rng = np.random.default_rng(500 + T)
    xn2 = rng.standard_normal((T, 512)).astype(np.float32)
    res = rng.standard_normal((T, 512)).astype(np.float32)       # fp32 residual (x1)
    if dt == "bf16":
        xn2 = S.round_to_bf16(xn2)
    idx, wts = random_topk(rng, T)
    if kind == "skewed":
        idx[:, 0] = 0
        idx[:, 1] = np.where(rng.random(T) < 0.8, 1, rng.integers(2, 8, T))
    w = _weights(501, dt)
    td = BF if dt == "bf16" else F32
    ws = poisoned_workspace(T, 1, dt)
    out = torch.full((T, 512), float("nan"), dtype=td, device="cuda")
    ptl.moe(dev(xn2, td), dev(idx, torch.int32), dev(wts, F32), dev(res, F32), out,
            ptl.to_device_layer(w, dt), ws)
    torch.cuda.synchronize()
    assert ptl.last_device_error(ws) == 0
    moe, _, _ = O.moe_routed(xn2, idx, wts, w["w1"], w["b1"], w["w2"], w["b2"])
    tol = (ATOL_BF16, RL2_BF16) if dt == "bf16" else (ATOL_F32, 1e-5)
    assert_close(host(out), res + moe, *tol, what=f"moe {dt} {kind}")


@pytest.mark.parametrize("dt,T", [("bf16", 1), ("bf16", 6823), ("fp32", 300)])
def test_head(dt, T):
    rng = np.random.default_rng(600 + T)
    h = rng.standard_normal((T, 512)).astype(np.float32) * 2
    if dt == "bf16":
        h = S.round_to_bf16(h)
    hw = {"lnf_g": rng.standard_normal(512).astype(np.float32) * 0.1 + 1,
          "lnf_b": rng.standard_normal(512).astype(np.float32) * 0.1,
          "w": rng.standard_normal(512).astype(np.float32) * 0.3,
          "b": np.array([0.3], np.float32)}
    mask = (rng.random(T) < 0.3).astype(np.uint8)
    mask[0] = 1
    td = BF if dt == "bf16" else F32
    ws = poisoned_workspace(T, 1, dt)
    probs = torch.full((T,), -1.0, dtype=F32, device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    ptl.head(dev(h, td), ptl.to_device_head(hw), dev(mask, torch.uint8), probs, n, ws)
    torch.cuda.synchronize()
    ref = O.head_forward(h, hw, mask)
    assert int(n.item()) == ref.size
    assert_close(host(probs)[:ref.size], ref, 1e-4, 1e-4, what="head probs")
    # logits beyond +-15 saturate at sigmoid(+-15)
    big = dict(hw, w=hw["w"] * 1000)
    ptl.head(dev(h, td), ptl.to_device_head(big), dev(mask, torch.uint8), probs, n, ws)
    torch.cuda.synchronize()
    pr = host(probs)[:ref.size]
    ref_big = O.head_forward(h, big, mask)
    assert np.sum(np.abs(ref_big - 0.5) > 0.4999996) > 0, "case must reach the clamp"
    assert_close(pr, ref_big, 1e-3, 1e-3, what="clamped head")
