"""Failure detection on the GPU without a fault: a kernel's bounded wait is
made to run out on purpose (an mbarrier phase nobody completes, a flag
nobody raises), the host reads PTL_ERR_TIMEOUT from the workspace error word,
and the same context and workspace then run a layer that matches the oracle."""
import pytest
import torch

from oracle import ptl_oracle as O
from packed_sequence_transformer_b200 import ptl
from packed_sequence_transformer_b200 import synthetic as S
from tests.gpu_util import assert_close, dev, host, tdt

pytestmark = pytest.mark.gpu

LIMIT_NS = 2_000_000  # 2 ms


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    ptl.lib()


@pytest.mark.parametrize("which", [0, 1], ids=["mbarrier", "flag"])
def test_bounded_wait_reports_timeout_and_context_survives(which):
    c = S.make_case("timeout_then_layer", lengths=[5, 130, 1], seed=3, dtype="fp32", gate_std=0.1)
    T, U = c.total_tokens, c.num_users
    ws = ptl.alloc_workspace(T, U, "fp32")
    assert ptl.last_device_error(ws) == 0
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    ptl.wait_selftest(ws, which, LIMIT_NS)
    t1.record()
    assert ptl.last_device_error(ws) == ptl.STATUS_CODE["PTL_ERR_TIMEOUT"]
    # the kernel waited out its limit before giving up, then returned
    assert t0.elapsed_time(t1) >= 0.9 * LIMIT_NS / 1e6
    # the error word was cleared by the read; the context is still usable
    assert ptl.last_device_error(ws) == 0
    x = dev(c.x, tdt("fp32"))
    out = torch.empty_like(x)
    ptl.layer_forward(x, out, dev(c.cu_seqlens, torch.int32),
                      ptl.to_device_layer(c.layers[0], "fp32"), ws)
    torch.cuda.synchronize()
    assert ptl.last_device_error(ws) == 0
    ref, it = O.layer_forward(c.x, c.cu_seqlens, c.layers[0], return_intermediates=True)
    unique = (it["gap"] > 1e-3) & (it["gap12"] > 1e-3)  # top-2 choice not near a tie
    assert unique.sum() > T // 2
    assert_close(host(out)[unique], ref[unique], 1e-4, 1e-5, what="layer after a timeout")
