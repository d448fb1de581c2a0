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


class NearTieChooser:
    """choose(layer, p, idx) hook for the oracle: where the GPU picked another
    top-2 pair (or slot order) than the oracle, follow the GPU's branch if
    and only if it is a valid choice in the oracle's own probabilities --
    both chosen experts within `margin` of the 2nd-largest probability, and
    slot 0 not below slot 1 by more than `margin`.  Any other difference is
    recorded as a violation: the result there is unique and must match."""

    def __init__(self, gpu_idx_per_layer, margin, later_margin=None):
        self.gpu = [np.asarray(g) for g in gpu_idx_per_layer]
        self.margin = margin
        self.later_margin = margin if later_margin is None else later_margin
        self.violations = []
        self.followed = []

    def __call__(self, layer, p, idx):
        g = self.gpu[layer]
        diff = np.any(g != idx, axis=1)
        if not diff.any():
            self.followed.append(0)
            return idx
        margin = self.margin if layer == 0 else self.later_margin
        ps = -np.sort(-p, axis=1)
        pg = np.take_along_axis(p, g, axis=1)
        valid = np.all(pg >= ps[:, 1:2] - margin, axis=1) & (pg[:, 0] >= pg[:, 1] - margin)
        valid &= g[:, 0] != g[:, 1]
        bad = diff & ~valid
        if bad.any():
            gap = (ps[:, 1] - ps[:, 2])[bad]
            self.violations.append((layer, np.where(bad)[0][:10].tolist(), int(bad.sum()),
                                    float(gap.max())))
        use = diff & valid
        self.followed.append(int(use.sum()))
        out = idx.copy()
        out[use] = g[use]
        return out

    def assert_ok(self):
        assert not self.violations, f"top-2 choices that are not near-ties differ: {self.violations}"
