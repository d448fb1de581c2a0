"""RepEncoder front end on the GPU (``ptl_rep_encoder``, both builds) against
the oracle on the same seeded inputs: bags of 0..4 ids over 28 tables, token
counts that span several 256-row tiles with a ragged tail, random LayerNorm
affine and bias; out-of-table ids are reported."""
import numpy as np
import pytest
import torch

from oracle import ptl_oracle as O
from packed_sequence_transformer_b200 import ptl
from packed_sequence_transformer_b200 import synthetic as S
from tests.gpu_util import assert_close, dev, host

pytestmark = pytest.mark.gpu

# bf16: the normalised rows are stored in bf16 (the oracle's bf16 storage
# mode rounds them the same way), products accumulate in fp32 over 14336,
# and the output (|v| up to ~16 here) takes one bf16 rounding, <= 2^-9 |v|.
TOL = {"bf16": (4e-2, 1e-2), "fp32": (2e-4, 1e-5)}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    ptl.lib()


def _device(c):
    td = torch.bfloat16 if c.dtype == "bf16" else torch.float32
    tables = [dev(t, td) for t in c.tables]
    keep = dict(tables=tables, ln_g=dev(c.ln_g, torch.float32), ln_b=dev(c.ln_b, torch.float32),
                w=dev(c.w, td), b=None if c.b is None else dev(c.b, torch.float32))
    st = ptl.rep_weights_struct(keep["tables"], keep["ln_g"], keep["ln_b"], keep["w"], keep["b"])
    return st, keep, td


def _run(c):
    st, keep, td = _device(c)
    T = c.num_tokens
    ws = ptl.rep_encoder_workspace(T, c.dtype)
    out = torch.full((T, 512), float("nan"), dtype=td, device="cuda")
    ids = dev(c.ids, torch.int64)
    off = dev(c.bag_offsets, torch.int64)
    ptl.rep_encoder(ids, off, T, st, out, ws)
    torch.cuda.synchronize()
    return out, ws


@pytest.mark.parametrize("dt,T", [("bf16", 1), ("bf16", 300), ("bf16", 1000), ("fp32", 1), ("fp32", 300)])
def test_rep_encoder_matches_oracle(dt, T):
    c = S.make_rep_case("rep", T, vocab=3000, max_bag=4, seed=40 + T, dtype=dt, random_affine=True)
    out, ws = _run(c)
    assert ptl.last_device_error(ws) == 0
    ref = O.rep_encoder(c.tables, c.ids, c.bag_offsets, T, c.ln_g, c.ln_b, c.w, c.b,
                        storage="bf16" if dt == "bf16" else None)
    assert_close(host(out), ref, *TOL[dt], what=f"rep encoder {dt} T={T}")


def test_all_bags_empty_gives_the_affine_shift():
    c = S.make_rep_case("rep_empty", 3, vocab=10, max_bag=2, empty_p=1.0, seed=5, dtype="fp32",
                        random_affine=True)
    assert c.ids.size == 0
    out, ws = _run(c)
    assert ptl.last_device_error(ws) == 0
    # every sum is 0, so the normalised row is ln_b and out = ln_b W^T + b
    want = c.ln_b.astype(np.float64) @ c.w.astype(np.float64).T + c.b
    assert_close(host(out), np.broadcast_to(want, (3, 512)), 2e-4, 1e-5, what="empty bags")


def test_out_of_table_id_is_reported():
    c = S.make_rep_case("rep_bad", 4, vocab=20, max_bag=3, empty_p=0.0, seed=6, dtype="bf16")
    c.ids[5] = 10_000
    out, ws = _run(c)
    assert ptl.last_device_error(ws) == ptl.STATUS_CODE["PTL_ERR_BAD_IDS"]
