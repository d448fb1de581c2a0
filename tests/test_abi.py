"""The C ABI library loads, exports every entry point include/ptl.h declares,
and rejects bad arguments on the host before touching the GPU.  CPU only:
no call here reaches a CUDA runtime function."""
import ctypes
import os
import re

import pytest

from packed_sequence_transformer_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def P():
    B.build()
    from packed_sequence_transformer_b200 import ptl
    ptl.lib()
    return ptl


def _declared():
    txt = open(os.path.join(ROOT, "include", "ptl.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(ptl_[a-z0-9_]+)\s*\(", txt)))


def test_exports_every_declared_symbol(P):
    names = _declared()
    assert len(names) >= 13
    for n in names:
        assert hasattr(P.lib(), n), n
    assert set(names) == set(P._SIGS), "binding and header disagree"


def test_status_strings_and_version(P):
    assert P.version() == 102
    for code in range(10):
        assert P.status_string(code)
    assert P.status_string(99) == "unknown status"


def test_workspace_size(P):
    a = P.workspace_size(6823, 60, "bf16")
    b = P.workspace_size(6823, 60, "fp32")
    assert a > 0 and b > a
    assert P.workspace_size(44000, 390, "bf16") > a
    assert P.workspace_size(-1, 1, "bf16") == 0
    assert P.workspace_size(10, 0, "bf16") == 0
    assert P.workspace_size(2 ** 31, 1, "bf16") == 0
    assert P.lib().ptl_workspace_size(10, 1, 7) == 0


FAKE = 0x10000          # aligned, never dereferenced: validation fails first
FAKE_MIS = 0x10008      # 8-byte aligned only


def _w(P, **over):
    s = P.LayerWeights()
    for n in P.LAYER_FIELDS:
        setattr(s, n, FAKE)
    for k, v in over.items():
        setattr(s, k, v)
    return s


def _layer(P, x=FAKE, out=FAKE + 4096, cu=FAKE, U=2, T=100, dt=1, w=None, ws=FAKE, wsb=None):
    L = P.lib()
    w = w or _w(P)
    wsb = P.workspace_size(max(T, 1), max(U, 1), dt if dt in (0, 1) else 1) if wsb is None else wsb
    return L.ptl_layer_forward(x, out, cu, U, T, dt, ctypes.byref(w), ws, wsb, None, None)


def test_host_validation_statuses(P):
    S = P.STATUS_CODE
    assert _layer(P, T=0) == S["PTL_OK"]                     # nothing to do, no launch
    assert _layer(P, x=None) == S["PTL_ERR_NULL"]
    assert _layer(P, cu=None) == S["PTL_ERR_NULL"]
    assert _layer(P, x=FAKE_MIS) == S["PTL_ERR_ALIGN"]
    assert _layer(P, ws=FAKE + 128) == S["PTL_ERR_ALIGN"]
    assert _layer(P, ws=None) == S["PTL_ERR_NULL"]
    assert _layer(P, dt=5) == S["PTL_ERR_DTYPE"]
    assert _layer(P, U=0) == S["PTL_ERR_SHAPE"]
    assert _layer(P, T=-3) == S["PTL_ERR_SHAPE"]
    assert _layer(P, T=2 ** 31) == S["PTL_ERR_SHAPE"]
    assert _layer(P, wsb=1000) == S["PTL_ERR_WORKSPACE"]
    assert _layer(P, out=FAKE) == S["PTL_ERR_SHAPE"]         # x aliases out
    assert _layer(P, w=_w(P, w_qkv=None)) == S["PTL_ERR_NULL"]
    assert _layer(P, x=None, T=0) == S["PTL_OK"]              # T = 0: pointers unused
    assert _layer(P, w=_w(P, w1=FAKE_MIS)) == S["PTL_ERR_ALIGN"]


def test_step_entry_points_validate(P):
    L = P.lib()
    S = P.STATUS_CODE
    w = _w(P)
    ws_b = P.workspace_size(64, 4, 1)
    assert L.ptl_attention(FAKE, FAKE, None, 4, 64, 1, FAKE, ws_b, None) == S["PTL_ERR_NULL"]
    assert L.ptl_attention(FAKE, FAKE, FAKE, 4, 0, 1, FAKE, ws_b, None) == S["PTL_OK"]
    assert L.ptl_gate(FAKE, FAKE, None, FAKE, 64, 1, ctypes.byref(w), FAKE, ws_b, None) == S["PTL_ERR_NULL"]
    assert L.ptl_route_build(FAKE + 2, 64, FAKE, FAKE, FAKE, ws_b, None) == S["PTL_ERR_ALIGN"]
    assert L.ptl_moe(FAKE, FAKE, FAKE, FAKE, FAKE, 64, 1, ctypes.byref(w), FAKE, 16, None) == S["PTL_ERR_WORKSPACE"]
    assert L.ptl_qkv_projection(FAKE, FAKE, 64, 3, ctypes.byref(w), FAKE, ws_b, None) == S["PTL_ERR_DTYPE"]
    h = P.HeadWeights(FAKE, FAKE, None, None)
    assert L.ptl_head(FAKE, ctypes.byref(h), FAKE, FAKE, None, 64, 1, FAKE, ws_b, None) == S["PTL_ERR_NULL"]
    arr = (P.LayerWeights * 2)(w, w)
    assert L.ptl_stack_forward(FAKE, FAKE + 4096, FAKE, 4, 64, 0, 1, arr, None, None, None, None,
                               FAKE, ws_b, None) == S["PTL_ERR_SHAPE"]
    assert L.ptl_last_device_error(None, 0, None) == S["PTL_ERR_NULL"]


def test_wait_selftest_host_checks(P):
    L = P.lib()
    S = P.STATUS_CODE
    assert L.ptl_wait_selftest(None, 256, 0, 10**6, None) == S["PTL_ERR_NULL"]
    assert L.ptl_wait_selftest(FAKE + 16, 256, 0, 10**6, None) == S["PTL_ERR_ALIGN"]
    assert L.ptl_wait_selftest(FAKE, 128, 0, 10**6, None) == S["PTL_ERR_WORKSPACE"]
    assert L.ptl_wait_selftest(FAKE, 256, 2, 10**6, None) == S["PTL_ERR_SHAPE"]
    assert L.ptl_wait_selftest(FAKE, 256, 1, 10, None) == S["PTL_ERR_SHAPE"]
    assert L.ptl_wait_selftest(FAKE, 256, 1, 2 * 10**9, None) == S["PTL_ERR_SHAPE"]


def test_runner_bucket_and_host_checks(P):
    L = P.lib()
    S = P.STATUS_CODE
    # 512-token buckets; padding users of <= 128 tokens: ceil(511 / 128) = 4 extra users
    assert P.runner_bucket(6823, 60) == (7168, 64)
    assert P.runner_bucket(7168, 60) == (7168, 64)
    assert P.runner_bucket(1, 1) == (512, 5)
    assert P.runner_bucket(0, 1) == (0, 5)
    assert P.runner_bucket(129, 3, 128) == (256, 4)
    assert P.runner_bucket(1000, 3, 1024) == (1024, 11)
    b, u = ctypes.c_int64(), ctypes.c_int32()
    for bad in [(100, 4, 96), (100, 0, 0), (-1, 4, 0), (2**31 - 1, 4, 0)]:
        assert L.ptl_runner_bucket(*bad, ctypes.byref(b), ctypes.byref(u)) == S["PTL_ERR_SHAPE"]
    assert L.ptl_runner_bucket(100, 4, 0, None, ctypes.byref(u)) == S["PTL_ERR_NULL"]
    w = _w(P)
    arr = (P.LayerWeights * 1)(w)
    r = ctypes.c_void_p()
    assert L.ptl_runner_create(1000, 4, 1, 1, arr, None, 0, None) == S["PTL_ERR_NULL"]
    assert L.ptl_runner_create(1000, 4, 1, 7, arr, None, 0, ctypes.byref(r)) == S["PTL_ERR_DTYPE"]
    assert L.ptl_runner_create(1000, 4, 0, 1, arr, None, 0, ctypes.byref(r)) == S["PTL_ERR_SHAPE"]
    assert L.ptl_runner_create(1000, 4, 1, 1, arr, None, 100, ctypes.byref(r)) == S["PTL_ERR_SHAPE"]
    assert r.value is None
    assert L.ptl_runner_forward(None, FAKE, FAKE, FAKE, 1, 10, None, None, None, None) == S["PTL_ERR_NULL"]
    assert L.ptl_runner_capture(None, 10) == S["PTL_ERR_NULL"]
    assert L.ptl_runner_last_device_error(None, None) == S["PTL_ERR_NULL"]
    assert L.ptl_runner_graphs(None) == -1
    L.ptl_runner_destroy(None)


def test_attention_masked_host_checks(P):
    L = P.lib()
    S = P.STATUS_CODE
    ws_b = P.workspace_size(64, 4, 1)
    m = P.AttnMaskStruct(1, None, None, 1, 0)
    assert L.ptl_attention_masked(FAKE, FAKE, FAKE, 4, 64, 1, None, FAKE, ws_b, None) == S["PTL_ERR_NULL"]
    bad_group = P.AttnMaskStruct(1, None, None, 0, 0)
    assert L.ptl_attention_masked(FAKE, FAKE, FAKE, 4, 64, 1, ctypes.byref(bad_group), FAKE, ws_b,
                                  None) == S["PTL_ERR_BAD_MASK"]
    bad_causal = P.AttnMaskStruct(2, None, None, 1, 0)
    assert L.ptl_attention_masked(FAKE, FAKE, FAKE, 4, 64, 1, ctypes.byref(bad_causal), FAKE, ws_b,
                                  None) == S["PTL_ERR_BAD_MASK"]
    assert L.ptl_attention_masked(FAKE, FAKE, FAKE, 4, 0, 1, ctypes.byref(m), FAKE, ws_b,
                                  None) == S["PTL_OK"]
    mis = P.AttnMaskStruct(1, FAKE + 2, None, 1, 0)
    assert L.ptl_attention_masked(FAKE, FAKE, FAKE, 4, 64, 1, ctypes.byref(mis), FAKE, ws_b,
                                  None) == S["PTL_ERR_ALIGN"]
    assert P.status_string(S["PTL_ERR_BAD_MASK"]).startswith("attention mask")


def test_rep_encoder_host_checks(P):
    L = P.lib()
    S = P.STATUS_CODE
    assert L.ptl_rep_encoder_workspace_size(100, 1) == 256 + ((100 * 14336 * 2 + 255) // 256) * 256
    assert L.ptl_rep_encoder_workspace_size(-1, 1) == 0
    assert L.ptl_rep_encoder_workspace_size(10, 5) == 0
    w = P.RepWeightsStruct()
    for i in range(28):
        w.tables[i] = FAKE
        w.vocab[i] = 10
    w.ln_g = w.ln_b = w.w = FAKE
    ws_b = L.ptl_rep_encoder_workspace_size(64, 1)
    ok = ctypes.byref(w)
    assert L.ptl_rep_encoder(FAKE, 10, FAKE, 64, 7, ok, FAKE, FAKE, ws_b, None) == S["PTL_ERR_DTYPE"]
    assert L.ptl_rep_encoder(FAKE, 10, None, 64, 1, ok, FAKE, FAKE, ws_b, None) == S["PTL_ERR_NULL"]
    assert L.ptl_rep_encoder(FAKE, 10, FAKE, 64, 1, ok, FAKE, FAKE, 16, None) == S["PTL_ERR_WORKSPACE"]
    assert L.ptl_rep_encoder(FAKE, 10, FAKE, 64, 1, ok, FAKE + 8, FAKE, ws_b, None) == S["PTL_ERR_ALIGN"]
    assert L.ptl_rep_encoder(FAKE, 10, FAKE, 0, 1, ok, FAKE, FAKE, ws_b, None) == S["PTL_OK"]
    w.vocab[3] = -1
    assert L.ptl_rep_encoder(FAKE, 10, FAKE, 64, 1, ok, FAKE, FAKE, ws_b, None) == S["PTL_ERR_SHAPE"]
    w.vocab[3] = 10
    w.tables[4] = None
    assert L.ptl_rep_encoder(FAKE, 10, FAKE, 64, 1, ok, FAKE, FAKE, ws_b, None) == S["PTL_ERR_NULL"]


def test_version_matches_header(P):
    hdr = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "ptl.h")).read()
    assert P.lib().ptl_version() == int(re.search(r"#define PTL_VERSION (\d+)", hdr).group(1)) == 102
