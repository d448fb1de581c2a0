"""ptl_attention_noalloc: the attention entry point for callers that cannot
allocate device memory (a host that owns all device memory through its own
pool and hands the library no allocator, or a latency-critical loop that
cannot afford cudaMalloc's possible device-wide synchronisation).  Its scratch
lives in a fixed array inside the library, so it takes no workspace.

Each call is checked against ptl_attention (the same kernels with a caller
workspace) on the same seeded inputs: the two run identical arithmetic, so
the outputs must agree bit for bit, in both builds, on two calls in a row,
at the array's exact size limit, and without the second call reserving any
device memory.  This file is collected last so that a run stopping at the
first failure has already run every other test; it also passes alone in a
fresh process."""
import numpy as np
import pytest
import torch

from packed_sequence_transformer_b200 import ptl
from packed_sequence_transformer_b200 import synthetic as S
from tests.gpu_util import dev, host

pytestmark = pytest.mark.gpu

MAX_TOKENS = 65536   # PTL_NOALLOC_MAX_TOKENS
MAX_USERS = 4096     # PTL_NOALLOC_MAX_USERS


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    ptl.lib()


def _attention_both(lengths, seed, dtype="bf16"):
    cu = S.offsets_from_lengths(lengths)
    T = int(cu[-1])
    qkv = np.random.default_rng(seed).standard_normal((T, 1536)).astype(np.float32)
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    q = dev(qkv, td)
    cu_d = dev(cu, torch.int32)
    ws = ptl.alloc_workspace(T, len(lengths), dtype)
    ref = torch.empty(T, 512, dtype=td, device="cuda")
    ptl.attention(q, ref, cu_d, ws)
    out = torch.full((T, 512), float("nan"), dtype=td, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    ptl.attention_noalloc(q, out, cu_d, device_status=status)
    torch.cuda.synchronize()
    assert ptl.last_device_error(ws) == 0
    assert int(status.item()) == 0
    return host(out), host(ref)


def _free_device_bytes():
    return torch.cuda.mem_get_info()[0]


def test_noalloc_attention_matches_workspace_attention_twice():
    # first call: the 60-user / 6823-token packing; second call: a ragged
    # packing with empty users and tile-boundary lengths, so a stale work list
    # from the first call would show
    first = _attention_both(S.config1_lengths(), seed=31)
    second = _attention_both([1, 127, 128, 129, 0, 300, 5, 513, 0], seed=32)
    for out, ref in (first, second):
        assert np.all(np.isfinite(out))
        np.testing.assert_array_equal(out, ref)


def test_noalloc_fp32_build_matches_workspace_attention():
    for lengths, seed in (([3, 7, 12, 20], 33), ([0, 200, 1, 129], 34)):
        out, ref = _attention_both(lengths, seed, dtype="fp32")
        assert np.all(np.isfinite(out))
        np.testing.assert_array_equal(out, ref)


def test_noalloc_at_its_size_limit_and_second_call_reserves_nothing():
    """Exactly PTL_NOALLOC_MAX_TOKENS tokens in PTL_NOALLOC_MAX_USERS users:
    the work list fills the array to its stated bound.  The call after the
    first reserves no device memory (free bytes and torch's allocator
    unchanged)."""
    lengths = np.full(MAX_USERS, MAX_TOKENS // MAX_USERS)
    lengths[0::2] += 3
    lengths[1::2] -= 3
    assert lengths.sum() == MAX_TOKENS and lengths.min() >= 0
    out, ref = _attention_both(lengths, seed=35)
    np.testing.assert_array_equal(out, ref)
    cu = dev(S.offsets_from_lengths(lengths), torch.int32)
    q = torch.zeros(MAX_TOKENS, 1536, dtype=torch.bfloat16, device="cuda")
    o = torch.empty(MAX_TOKENS, 512, dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    free0, alloc0 = _free_device_bytes(), torch.cuda.memory_allocated()
    for _ in range(2):
        ptl.attention_noalloc(q, o, cu)
    torch.cuda.synchronize()
    assert _free_device_bytes() == free0
    assert torch.cuda.memory_allocated() == alloc0


def test_noalloc_rejects_sizes_beyond_its_array():
    L = ptl.lib()
    # host-side rejection: nothing is launched, the pointers are never used
    too_many_tokens = L.ptl_attention_noalloc(0x10000, 0x20000, 0x30000, 4, MAX_TOKENS + 1, 1,
                                              None, None)
    too_many_users = L.ptl_attention_noalloc(0x10000, 0x20000, 0x30000, MAX_USERS + 1, 100, 1,
                                             None, None)
    assert too_many_tokens == ptl.STATUS_CODE["PTL_ERR_SHAPE"]
    assert too_many_users == ptl.STATUS_CODE["PTL_ERR_SHAPE"]


def test_noalloc_reports_bad_offsets():
    cu = np.array([0, 9, 4, 20], np.int64)
    qkv = torch.zeros(20, 1536, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(20, 512, dtype=torch.bfloat16, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    ptl.attention_noalloc(qkv, out, dev(cu, torch.int32), device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == ptl.STATUS_CODE["PTL_ERR_BAD_OFFSETS"]
