"""ptl_partition_users (host code of libptl, no GPU): one batch's users split
into contiguous ranges, one per GPU, minimising the largest range's cost.
Checked against an exhaustive search over every contiguous split on small
batches and a dynamic programme on the 60-user packing, plus coverage,
ordering and the host-side rejections."""
import itertools

import numpy as np
import pytest

from packed_sequence_transformer_b200 import ptl
from packed_sequence_transformer_b200 import synthetic as S

GEMM_FLOPS_PER_TOKEN = 2 * 512 * 1536 + 2 * 512 * 512 + 2 * 512 * 8 + 2 * 2 * (2 * 512 * 1024)


def cost(L):
    """A user's work: one layer's GEMM FLOPs for its tokens plus its causal
    attention FLOPs (QK^T and PV over 8 heads of 64)."""
    L = int(L)
    return GEMM_FLOPS_PER_TOKEN * L + 2048 * (L * (L + 1) // 2)


def part_costs(lengths, begin):
    return [sum(cost(L) for L in lengths[begin[r]:begin[r + 1]]) for r in range(len(begin) - 1)]


def best_exhaustive(lengths, parts):
    U = len(lengths)
    best = None
    for cuts in itertools.combinations_with_replacement(range(U + 1), parts - 1):
        begin = [0, *cuts, U]
        m = max(part_costs(lengths, begin))
        best = m if best is None else min(best, m)
    return best


def best_dp(lengths, parts):
    U = len(lengths)
    pre = np.concatenate([[0], np.cumsum([cost(L) for L in lengths])])
    INF = float("inf")
    dp = [[INF] * (U + 1) for _ in range(parts + 1)]
    dp[0][0] = 0
    for p in range(1, parts + 1):
        for u in range(U + 1):
            dp[p][u] = min(max(dp[p - 1][v], pre[u] - pre[v]) for v in range(u + 1))
    return dp[parts][U]


def check_shape(begin, U, parts):
    assert len(begin) == parts + 1 and begin[0] == 0 and begin[-1] == U
    assert np.all(np.diff(begin) >= 0)


@pytest.mark.parametrize("seed", range(30))
def test_optimal_against_every_contiguous_split(seed):
    rng = np.random.default_rng(seed)
    U = int(rng.integers(1, 8))
    lengths = rng.integers(0, 300, size=U)
    parts = int(rng.integers(1, 5))
    begin = ptl.partition_users(S.offsets_from_lengths(lengths), parts)
    check_shape(begin, U, parts)
    assert max(part_costs(lengths, begin)) == best_exhaustive(lengths, parts)


@pytest.mark.parametrize("parts", [1, 2, 3, 4, 8])
def test_packing_split_is_optimal_and_covers_every_user(parts):
    lengths = S.config1_lengths()
    begin = ptl.partition_users(S.offsets_from_lengths(lengths), parts)
    check_shape(begin, len(lengths), parts)
    costs = part_costs(lengths, begin)
    assert max(costs) == best_dp(lengths, parts)
    assert sum(costs) == sum(cost(L) for L in lengths)
    owner = np.repeat(np.arange(parts), np.diff(begin))
    assert owner.size == len(lengths)                      # each user once, in order


def test_more_parts_than_users_leaves_trailing_parts_empty():
    begin = ptl.partition_users([0, 5, 5, 9], 6)
    check_shape(begin, 3, 6)
    assert max(part_costs([5, 0, 4], begin)) == cost(5)


def test_rejections():
    code = ptl.STATUS_CODE
    with pytest.raises(ptl.PtlError) as e:
        ptl.partition_users([0, 5, 3], 2)
    assert e.value.status == code["PTL_ERR_BAD_OFFSETS"]
    with pytest.raises(ptl.PtlError) as e:
        ptl.partition_users([1, 5], 2)
    assert e.value.status == code["PTL_ERR_BAD_OFFSETS"]
    with pytest.raises(ptl.PtlError) as e:
        ptl.partition_users([0, 5], 0)
    assert e.value.status == code["PTL_ERR_SHAPE"]
