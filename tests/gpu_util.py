"""Helpers shared by the GPU parity tests: upload seeded cases, compare."""
import numpy as np
import torch

from packed_sequence_transformer_b200 import ptl
from packed_sequence_transformer_b200 import synthetic as S


def dev(a, dtype, device="cuda"):
    return torch.as_tensor(np.ascontiguousarray(a)).to(device=device, dtype=dtype).contiguous()


def host(t):
    return t.detach().to("cpu", torch.float64).numpy() if t.is_floating_point() else t.cpu().numpy()


def tdt(case_dtype):
    return torch.bfloat16 if case_dtype == "bf16" else torch.float32


def poisoned_workspace(T, U, dtype):
    """Workspace filled with 0xFF bytes (NaN floats, -1 ints) so that a read of
    anything the kernels did not write shows up as a mismatch."""
    ws = ptl.alloc_workspace(T, U, dtype)
    ws.fill_(255)
    return ws


def max_abs(a, b):
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64)))) if np.size(a) else 0.0


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def assert_close(gpu, ref, atol, rl2, what=""):
    g = np.asarray(gpu, np.float64)
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    ma, r = max_abs(g, ref), rel_l2(g, ref)
    assert ma <= atol and r <= rl2, f"{what}: max-abs {ma:.3e} (<= {atol}), rel-L2 {r:.3e} (<= {rl2})"
    return ma, r


def subset_users(case: S.Case, users):
    """Rows and offsets of a subset of users (users are independent)."""
    cu = case.cu_seqlens
    rows = np.concatenate([np.arange(cu[u], cu[u + 1]) for u in users])
    sub_cu = S.offsets_from_lengths([cu[u + 1] - cu[u] for u in users])
    return rows, sub_cu


def random_topk(rng, T, E=8):
    """Distinct expert pairs per token with weights w0 >= w1, w0 + w1 = 1."""
    idx = np.stack([rng.choice(E, 2, replace=False) for _ in range(T)]).astype(np.int32)
    w0 = rng.uniform(0.5, 1.0, T).astype(np.float32)
    w = np.stack([w0, (1.0 - w0).astype(np.float32)], 1)
    return idx, w


def check_perm_is_stable_sort(idx, perm, off, E=8):
    """What is unique about the route order: a stable counting sort of r by idx[r]."""
    flat = np.asarray(idx).reshape(-1)
    expect = np.argsort(flat, kind="stable")
    cnt = np.bincount(flat, minlength=E)
    assert np.array_equal(np.asarray(off), np.concatenate([[0], np.cumsum(cnt)]))
    assert np.array_equal(np.asarray(perm), expect)


def routing_flips(g_idx, it, margin=1e-3):
    """Compare the GPU's top-2 choice with the oracle's.  Returns (setflip,
    ordflip) masks.  Enforces what is unique: the chosen pair must match
    wherever the oracle's 2nd-vs-3rd gap exceeds `margin`, and its slot order
    wherever the 1st-vs-2nd gap also does."""
    g_idx = np.asarray(g_idx)
    o_idx = np.asarray(it["idx"])
    setflip = np.any(np.sort(g_idx, 1) != np.sort(o_idx, 1), axis=1)
    ordflip = ~setflip & np.any(g_idx != o_idx, axis=1)
    bad_set = setflip & (it["gap"] > margin)
    bad_ord = ordflip & (it["gap12"] > margin)
    assert not bad_set.any(), f"top-2 pair differs on {int(bad_set.sum())} tokens with gap > {margin}"
    assert not bad_ord.any(), f"top-2 order differs on {int(bad_ord.sum())} tokens with gap > {margin}"
    return setflip, ordflip


def check_near_tie_choice(rows, g_idx, it, wts, gpu_rows, tol, margin=1e-3):
    """Where a near-tie let the GPU pick another pair, that pair must be a
    valid top-2 (both experts within `margin` of the 2nd-largest probability)
    and the GPU output must equal the oracle's layer output with that pair."""
    from oracle import ptl_oracle as O
    if len(rows) == 0:
        return
    p = it["p"][rows]
    pair = np.asarray(g_idx)[rows]
    p2 = -np.sort(-p, axis=1)[:, 1]
    chosen = np.take_along_axis(p, pair, axis=1)
    assert np.all(chosen >= p2[:, None] - margin), "GPU chose an expert far below the top-2"
    w = chosen / chosen.sum(1, keepdims=True)
    moe, _, _ = O.moe_routed(it["xn2"][rows], pair, w, wts["w1"], wts["b1"], wts["w2"], wts["b2"])
    assert_close(gpu_rows, it["x1"][rows] + moe, *tol, what="near-tie tokens")


def taint_mask(cu, flips_any):
    """Tokens whose user-causal context (itself or an earlier token of the
    same user) had a different top-2 pair at some layer."""
    taint = np.zeros(len(flips_any), bool)
    for u in range(len(cu) - 1):
        s, e = int(cu[u]), int(cu[u + 1])
        f = np.where(flips_any[s:e])[0]
        if f.size:
            taint[s + f.min():e] = True
    return taint
