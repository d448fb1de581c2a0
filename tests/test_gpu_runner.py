"""The bucketed CUDA-graph runner (``ptl_runner_*``) on the GPU: batches of
different sizes, padded to 512-token buckets with padding users, give the
real rows of a direct ``ptl_stack_forward`` call on the unpadded batch bit
for bit; a bucket's graph is captured once and replayed; host (pinned)
buffers work as inputs and outputs; malformed offsets are reported; and the
fp32 runner matches the fp64 oracle."""
import numpy as np
import pytest
import torch

from oracle import ptl_oracle as O
from packed_sequence_transformer_b200 import ptl
from packed_sequence_transformer_b200 import synthetic as S
from tests.gpu_util import assert_close, dev, host, tdt

pytestmark = pytest.mark.gpu

LENGTHS = [3, 130, 1, 0, 40, 257, 600, 12, 77, 128, 129, 5, 300, 1, 64, 200]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    ptl.lib()


@pytest.fixture(scope="module")
def case():
    return S.make_case("runner", lengths=LENGTHS, seed=11, dtype="bf16", num_layers=2,
                       gate_std=0.1, with_head=True)


def batch(c, a, b, dt):
    """Users a .. b-1 of the case as their own packed batch."""
    cu = np.asarray(c.cu_seqlens)
    r0, r1 = int(cu[a]), int(cu[b])
    return (dev(c.x[r0:r1], tdt(dt)), dev(cu[a:b + 1] - r0, torch.int32),
            dev(c.pred_mask[r0:r1], torch.uint8), (r0, r1))


def direct(c, x, cu, mask, layers, head):
    T, U = x.shape[0], cu.numel() - 1
    ws = ptl.alloc_workspace(T, U, "bf16")
    out = torch.empty_like(x)
    probs = torch.full((T,), float("nan"), device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    ptl.stack_forward(x, out, cu, layers, ws, head=head, pred_mask=mask, probs=probs, n_pred=n)
    torch.cuda.synchronize()
    assert ptl.last_device_error(ws) == 0
    return out, probs, n


def test_bucket_arithmetic():
    assert ptl.runner_bucket(6823, 60) == (7168, 64)
    assert ptl.runner_bucket(512, 60) == (512, 64)
    assert ptl.runner_bucket(513, 60, 128) == (640, 61)


def test_runner_equals_direct_call_bit_for_bit(case):
    c = case
    layers = [ptl.to_device_layer(w, "bf16") for w in c.layers]
    head = ptl.to_device_head(c.head)
    r = ptl.StackRunner(2400, 16, layers, "bf16", head=head)
    # users a .. b-1: T = 174 (bucket 512), 131 (512 again), 897 (1024),
    # 297 (512 again), all 1947 (2048), 1516 (1536)
    seen = set()
    for a, b in [(0, 5), (1, 4), (4, 8), (5, 7), (0, 16), (6, 16)]:
        x, cu, mask, _ = batch(c, a, b, "bf16")
        T = x.shape[0]
        if T == 0:
            continue
        out = torch.full_like(x, float("nan"))
        probs = torch.full((T,), float("nan"), device="cuda")
        n = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        r.forward(x, cu, out=out, pred_mask=mask, probs=probs, n_pred=n)
        torch.cuda.synchronize()
        assert r.last_device_error() == 0
        seen.add(ptl.runner_bucket(T, 16)[0])
        assert r.graphs() == len(seen)
        d_out, d_probs, d_n = direct(c, x, cu, mask, layers, head)
        assert torch.equal(out, d_out), f"users {a}..{b}: hidden rows differ"
        k = int(d_n.item())
        assert int(n.item()) == k == int(mask.sum().item())
        assert torch.equal(probs[:k], d_probs[:k]), f"users {a}..{b}: probs differ"
    r.close()


def test_runner_host_buffers_and_replay(case):
    c = case
    layers = [ptl.to_device_layer(w, "bf16") for w in c.layers]
    head = ptl.to_device_head(c.head)
    r = ptl.StackRunner(3000, 16, layers, "bf16", head=head)
    x, cu, mask, _ = batch(c, 0, 16, "bf16")
    T = x.shape[0]
    r.capture(T)
    assert r.graphs() == 1
    xh, cuh, mh = x.cpu().pin_memory(), cu.cpu().pin_memory(), mask.cpu().pin_memory()
    outs = []
    for _ in range(3):  # replays of the same bucket give the same answer
        out_h = torch.empty(T, 512, dtype=torch.bfloat16).pin_memory()
        probs_h = torch.empty(T, dtype=torch.float32).pin_memory()
        n_h = torch.zeros(1, dtype=torch.int32).pin_memory()
        r.forward(xh, cuh, out=out_h, pred_mask=mh, probs=probs_h, n_pred=n_h)
        torch.cuda.synchronize()
        assert r.last_device_error() == 0
        outs.append((out_h.clone(), probs_h[:int(n_h.item())].clone()))
    assert r.graphs() == 1
    d_out, d_probs, d_n = direct(c, x, cu, mask, layers, head)
    for o, p in outs:
        assert torch.equal(o, d_out.cpu())
        assert torch.equal(p, d_probs[:int(d_n.item())].cpu())
    # probabilities only: out may be omitted when there is a head
    probs = torch.empty(T, device="cuda")
    r.forward(x, cu, pred_mask=mask, probs=probs)
    torch.cuda.synchronize()
    assert torch.equal(probs[:int(d_n.item())], d_probs[:int(d_n.item())])
    r.close()


def test_two_runners_on_two_streams_overlap_and_agree(case):
    """The serving loop of the bench: two runners on two streams, batches
    alternating between them with no host synchronisation, so that one
    runner's copies and graph run while the other's graph does.  Every batch's
    rows and probabilities equal the direct call's bit for bit."""
    c = case
    layers = [ptl.to_device_layer(w, "bf16") for w in c.layers]
    head = ptl.to_device_head(c.head)
    x, cu, mask, _ = batch(c, 0, 16, "bf16")
    T = x.shape[0]
    d_out, d_probs, d_n = direct(c, x, cu, mask, layers, head)
    k = int(d_n.item())
    xh, cuh, mh = x.cpu().pin_memory(), cu.cpu().pin_memory(), mask.cpu().pin_memory()
    lanes = []
    for _ in range(2):
        r = ptl.StackRunner(T, 16, layers, "bf16", head=head)
        r.capture(T)
        lanes.append((r, torch.cuda.Stream()))
    results = []
    for i in range(6):
        r, s = lanes[i % 2]
        out_h = torch.empty(T, 512, dtype=torch.bfloat16).pin_memory()
        probs_h = torch.empty(T, dtype=torch.float32).pin_memory()
        n_h = torch.zeros(1, dtype=torch.int32).pin_memory()
        with torch.cuda.stream(s):
            r.forward(xh, cuh, out=out_h, pred_mask=mh, probs=probs_h, n_pred=n_h, stream=s)
        results.append((out_h, probs_h, n_h))
    torch.cuda.synchronize()
    for r, s in lanes:
        assert r.last_device_error(s) == 0
        r.close()
    for out_h, probs_h, n_h in results:
        assert int(n_h.item()) == k
        assert torch.equal(out_h, d_out.cpu())
        assert torch.equal(probs_h[:k], d_probs[:k].cpu())


def test_runner_limits_and_bad_offsets(case):
    c = case
    layers = [ptl.to_device_layer(w, "bf16") for w in c.layers]
    r = ptl.StackRunner(600, 4, layers, "bf16")
    x, cu, _, _ = batch(c, 0, 3, "bf16")  # 134 tokens, 3 users
    out = torch.empty_like(x)
    big = torch.zeros(601, 512, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ptl.PtlError):
        r.forward(big, dev(np.array([0, 601]), torch.int32), out=torch.empty_like(big))
    with pytest.raises(ptl.PtlError):
        r.forward(x, dev(np.array([0, 1, 2, 3, 4, 134]), torch.int32), out=out)
    # the last offset is not T: reported through the offsets validator
    bad = cu.clone()
    bad[-1] = x.shape[0] - 5
    r.forward(x, bad, out=out)
    assert r.last_device_error() == ptl.STATUS_CODE["PTL_ERR_BAD_OFFSETS"]
    # the same runner goes on with a good batch
    r.forward(x, cu, out=out)
    torch.cuda.synchronize()
    assert r.last_device_error() == 0
    d_out, _, _ = direct(c, x, cu, dev(np.ones(x.shape[0], np.uint8), torch.uint8), layers, None)
    assert torch.equal(out, d_out)
    r.close()


def test_fp32_runner_matches_oracle():
    """One fp32 layer + head through a 128-token-stride runner against the
    fp64 oracle, on the tokens whose top-2 choice is not near a tie."""
    c = S.make_case("runner_f32", lengths=[5, 130, 1, 60], seed=12, dtype="fp32", num_layers=1,
                    gate_std=0.1, with_head=True)
    layers = [ptl.to_device_layer(w, "fp32") for w in c.layers]
    head = ptl.to_device_head(c.head)
    r = ptl.StackRunner(1000, 8, layers, "fp32", head=head, stride=128)
    x = dev(c.x, torch.float32)
    cu = dev(c.cu_seqlens, torch.int32)
    mask = dev(c.pred_mask, torch.uint8)
    T = x.shape[0]
    out = torch.empty_like(x)
    probs = torch.empty(T, device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    r.forward(x, cu, out=out, pred_mask=mask, probs=probs, n_pred=n)
    torch.cuda.synchronize()
    assert r.last_device_error() == 0
    _, it = O.layer_forward(c.x, c.cu_seqlens, c.layers[0], return_intermediates=True)
    ok = (it["gap"] > 1e-3) & (it["gap12"] > 1e-3)
    assert ok.sum() > T // 2
    ref_h, ref_p = O.stack_forward(c.x, c.cu_seqlens, c.layers, c.head, c.pred_mask)
    assert_close(host(out)[ok], ref_h[ok], 1e-4, 1e-5, what="fp32 runner hidden")
    sel = np.asarray(c.pred_mask) != 0
    assert int(n.item()) == ref_p.size == int(sel.sum())
    ok_p = ok[sel]
    assert_close(host(probs)[:ref_p.size][ok_p], ref_p[ok_p], 1e-4, 1e-5, what="fp32 runner probs")
    r.close()
