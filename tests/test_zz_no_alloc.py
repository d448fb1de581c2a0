"""ptl_attention_noalloc: the attention entry point for callers that cannot
allocate device memory (their host owns all device memory, or cudaMalloc's
possible device-wide synchronisation is not acceptable).  Its scratch lives in
a fixed array inside the library, so it needs no workspace.  Two calls in a
row, each checked against ptl_attention (which uses a caller workspace) on the
same seeded inputs, within the tolerance of the other attention tests.  This
file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

from packed_sequence_transformer_b200 import ptl
from packed_sequence_transformer_b200 import synthetic as S
from tests.gpu_util import assert_close, dev, host

pytestmark = pytest.mark.gpu

ATOL_BF16 = 2e-2
RL2_BF16 = 1e-2
MAX_TOKENS = 65536   # PTL_NOALLOC_MAX_TOKENS
MAX_USERS = 4096     # PTL_NOALLOC_MAX_USERS


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    ptl.lib()


def _attention_both(lengths, seed):
    cu = S.offsets_from_lengths(lengths)
    T = int(cu[-1])
    qkv = S.round_to_bf16(np.random.default_rng(seed).standard_normal((T, 1536)).astype(np.float32))
    q = dev(qkv, torch.bfloat16)
    cu_d = dev(cu, torch.int32)
    ws = ptl.alloc_workspace(T, len(lengths), "bf16")
    ref = torch.empty(T, 512, dtype=torch.bfloat16, device="cuda")
    ptl.attention(q, ref, cu_d, ws)
    out = torch.full((T, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    ptl.attention_noalloc(q, out, cu_d, device_status=status)
    torch.cuda.synchronize()
    assert ptl.last_device_error(ws) == 0
    assert int(status.item()) == 0
    return host(out), host(ref)


def test_noalloc_attention_matches_workspace_attention_twice():
    # first call: the 60-user / 6823-token packing; second call: a ragged
    # packing with empty users and tile-boundary lengths, so a stale work list
    # from the first call would show
    first = _attention_both(S.config1_lengths(), seed=31)
    second = _attention_both([1, 127, 128, 129, 0, 300, 5, 513, 0], seed=32)
    for out, ref in (first, second):
        assert_close(out, ref, ATOL_BF16, RL2_BF16, what="noalloc attention")


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

