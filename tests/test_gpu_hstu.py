"""HSTU-style masked attention on the GPU (``ptl_attention_masked``, both
builds) against the oracle's masked attention on the same seeded inputs:
contextual tokens, candidate groups, sliding windows, the no-mask type and
their combination, over packings with empty users, single tokens and users
that straddle 128-token blocks; the default mask equals the causal
attention bit for bit; malformed per-user counts are reported."""
import numpy as np
import pytest
import torch

from oracle import ptl_oracle as O
from packed_sequence_transformer_b200 import ptl
from packed_sequence_transformer_b200 import synthetic as S
from tests.gpu_util import assert_close, dev, host, poisoned_workspace

pytestmark = pytest.mark.gpu

BF = torch.bfloat16
F32 = torch.float32
# as for the causal attention: one bf16 rounding of O(1) outputs plus fp32
# accumulation of bf16 products; fp32 differs from fp64 by fp32 rounding only
TOL = {"bf16": (2e-2, 1e-2), "fp32": (1e-4, 1e-5)}

LENGTHS = [1, 127, 128, 129, 0, 300, 5, 513, 0, 40, 260]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    ptl.lib()


def _counts(lengths, seed, frac_ctx, frac_tgt):
    """Per-user contextual and candidate counts that fit in each user."""
    rng = np.random.default_rng(seed)
    L = np.asarray(lengths)
    ctx = np.floor(rng.uniform(0, frac_ctx, len(L)) * L).astype(np.int32)
    tgt = np.floor(rng.uniform(0, frac_tgt, len(L)) * (L - ctx)).astype(np.int32)
    return ctx, tgt


MASKS = {
    "default": dict(),
    "no_mask": dict(causal=False),
    "context": dict(ctx=(0.6, 0.0)),
    "targets_g1": dict(ctx=(0.0, 0.4), group=1),
    "targets_g3": dict(ctx=(0.0, 0.5), group=3),
    "targets_one_group": dict(ctx=(0.0, 0.5), group=100000),
    "window_1": dict(window=1),
    "window_50": dict(window=50),
    "window_200_no_mask": dict(window=200, causal=False),
    "combined": dict(ctx=(0.3, 0.3), group=4, window=150),
    "combined_no_mask": dict(ctx=(0.3, 0.3), group=2, window=300, causal=False),
    "targets_small_window": dict(ctx=(0.2, 0.5), group=3, window=7),
    "targets_no_mask_g2": dict(ctx=(0.0, 0.6), group=2, causal=False),
}


def _run(dt, lengths, spec, seed=21):
    cu = S.offsets_from_lengths(lengths)
    T = int(cu[-1])
    rng = np.random.default_rng(seed)
    qkv = rng.standard_normal((T, 1536)).astype(np.float32)
    if dt == "bf16":
        qkv = S.round_to_bf16(qkv)
    td = BF if dt == "bf16" else F32
    ctx = tgt = None
    if "ctx" in spec:
        ctx, tgt = _counts(lengths, seed + 1, *spec["ctx"])
    causal = spec.get("causal", True)
    group = spec.get("group", 1)
    window = spec.get("window", 0)
    ws = poisoned_workspace(T, len(lengths), dt)
    out = torch.full((T, 512), float("nan"), dtype=td, device="cuda")
    ptl.attention_masked(dev(qkv, td), out, dev(cu, torch.int32), ws, causal=causal,
                         num_contexts=None if ctx is None else dev(ctx, torch.int32),
                         num_targets=None if tgt is None else dev(tgt, torch.int32),
                         target_group_size=group, window=window)
    torch.cuda.synchronize()
    assert ptl.last_device_error(ws) == 0
    q, k, v = O.split_qkv(qkv)
    ref = O.jagged_hstu_attention(q, k, v, cu, causal=causal, num_contexts=ctx, num_targets=tgt,
                                  target_group_size=group, window=window).reshape(T, 512)
    return out, ref, qkv, cu


@pytest.mark.parametrize("name", list(MASKS))
@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_masked_attention_matches_oracle(name, dt):
    out, ref, _, _ = _run(dt, LENGTHS, MASKS[name])
    assert_close(host(out), ref, *TOL[dt], what=f"masked attention {name} {dt}")


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_default_mask_equals_causal_attention(dt):
    out, _, qkv, cu = _run(dt, LENGTHS, MASKS["default"])
    td = BF if dt == "bf16" else F32
    ws = ptl.alloc_workspace(int(cu[-1]), len(LENGTHS), dt)
    plain = torch.empty_like(out)
    ptl.attention(dev(qkv, td), plain, dev(cu, torch.int32), ws)
    torch.cuda.synchronize()
    assert torch.equal(out, plain)


def test_window_one_outputs_own_v_rows():
    out, _, qkv, cu = _run("bf16", LENGTHS, MASKS["window_1"])
    assert torch.equal(out.cpu(), torch.from_numpy(qkv[:, 1024:]).to(BF))


def test_masked_attention_config1_packing():
    """The 60-user / 6823-token packing with every feature on (bf16)."""
    lengths = S.config1_lengths()
    out, ref, _, _ = _run("bf16", lengths, MASKS["combined"], seed=31)
    assert_close(host(out), ref, *TOL["bf16"], what="masked attention config1")


@pytest.mark.parametrize("bad", ["too_many", "negative"])
def test_bad_counts_are_reported(bad):
    lengths = [5, 10]
    cu = S.offsets_from_lengths(lengths)
    ctx = np.array([3, 4], np.int32)
    tgt = np.array([3, 2], np.int32) if bad == "too_many" else np.array([0, -1], np.int32)
    ws = ptl.alloc_workspace(15, 2, "bf16")
    qkv = torch.zeros(15, 1536, dtype=BF, device="cuda")
    out = torch.empty(15, 512, dtype=BF, device="cuda")
    ptl.attention_masked(qkv, out, dev(cu, torch.int32), ws, num_contexts=dev(ctx, torch.int32),
                         num_targets=dev(tgt, torch.int32))
    assert ptl.last_device_error(ws) == ptl.STATUS_CODE["PTL_ERR_BAD_MASK"]
    # the workspace serves a good call afterwards
    ptl.attention_masked(qkv, out, dev(cu, torch.int32), ws, num_contexts=dev(ctx, torch.int32))
    assert ptl.last_device_error(ws) == 0
