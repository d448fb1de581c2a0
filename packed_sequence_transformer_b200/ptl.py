"""Python binding of libptl (ctypes).  Argument marshalling only: every step
of the layer runs in the library's CUDA kernels.  torch provides device
memory and streams.

The functions mirror the C ABI in include/ptl.h (names without the ``ptl_``
prefix) and take torch tensors.  A status other than PTL_OK raises
``PtlError``.  If libptl.so is missing or cannot be loaded, every call
raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Iterable, List, Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libptl.so")

PTL_F32, PTL_BF16 = 0, 1
STATUS = {
    0: "PTL_OK", 1: "PTL_ERR_NULL", 2: "PTL_ERR_ALIGN", 3: "PTL_ERR_SHAPE",
    4: "PTL_ERR_BAD_OFFSETS", 5: "PTL_ERR_WORKSPACE", 6: "PTL_ERR_DTYPE", 7: "PTL_ERR_CUDA",
    8: "PTL_ERR_TIMEOUT", 9: "PTL_ERR_UNSUPPORTED", 10: "PTL_ERR_BAD_MASK", 11: "PTL_ERR_BAD_IDS",
}
STATUS_CODE = {v: k for k, v in STATUS.items()}

LAYER_FIELDS = ("ln1_g", "ln1_b", "w_qkv", "b_qkv", "w_o", "b_o", "ln2_g", "ln2_b", "w_gate",
                "b_gate", "w1", "b1", "w2", "b2")
HEAD_FIELDS = ("lnf_g", "lnf_b", "w", "b")
# Stored in float32 in both builds; the rest of a layer in the build dtype.
FP32_FIELDS = ("ln1_g", "ln1_b", "ln2_g", "ln2_b", "w_gate", "b_gate", "b_qkv", "b_o", "b1", "b2")


class PtlError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        self.name = STATUS.get(status, str(status))
        super().__init__(f"{where}: {self.name} ({status_string(status) if _lib else ''})")


class LayerWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in LAYER_FIELDS]


class HeadWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in HEAD_FIELDS]


class DebugOut(ctypes.Structure):
    _fields_ = [("topk_idx", ctypes.c_void_p), ("topk_w", ctypes.c_void_p),
                ("perm", ctypes.c_void_p), ("expert_off", ctypes.c_void_p)]


class AttnMaskStruct(ctypes.Structure):
    _fields_ = [("causal", ctypes.c_int32), ("num_contexts", ctypes.c_void_p),
                ("num_targets", ctypes.c_void_p), ("target_group_size", ctypes.c_int32),
                ("window", ctypes.c_int32)]


class RepWeightsStruct(ctypes.Structure):
    _fields_ = [("tables", ctypes.c_void_p * 28), ("vocab", ctypes.c_int64 * 28),
                ("ln_g", ctypes.c_void_p), ("ln_b", ctypes.c_void_p), ("w", ctypes.c_void_p),
                ("b", ctypes.c_void_p)]


class Trace(ctypes.Structure):
    _fields_ = [("events", ctypes.POINTER(ctypes.c_void_p)), ("kinds", ctypes.POINTER(ctypes.c_int32)),
                ("capacity", ctypes.c_int32), ("count", ctypes.c_int32)]


KERNEL_KINDS = {0: "clear", 1: "worklist", 2: "layernorm", 3: "gemm_qkv", 4: "attention",
                5: "gemm_out", 6: "gate", 7: "route", 8: "gemm_expert1", 9: "gemm_expert2",
                10: "head", 11: "copy", 12: "combine", 99: "end"}

_lib = None
_SIGS = {
    "ptl_version": ([], ctypes.c_int32),
    "ptl_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "ptl_workspace_size": ([ctypes.c_int64, ctypes.c_int32, ctypes.c_int], ctypes.c_size_t),
    "ptl_layer_forward": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                           ctypes.c_int64, ctypes.c_int, ctypes.POINTER(LayerWeights),
                           ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(DebugOut),
                           ctypes.c_void_p], ctypes.c_int),
    "ptl_stack_forward": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                           ctypes.c_int64, ctypes.c_int32, ctypes.c_int, ctypes.POINTER(LayerWeights),
                           ctypes.POINTER(HeadWeights), ctypes.c_void_p, ctypes.c_void_p,
                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p],
                          ctypes.c_int),
    "ptl_qkv_projection": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                            ctypes.POINTER(LayerWeights), ctypes.c_void_p, ctypes.c_size_t,
                            ctypes.c_void_p], ctypes.c_int),
    "ptl_attention": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                       ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t,
                       ctypes.c_void_p], ctypes.c_int),
    "ptl_attention_masked": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                              ctypes.c_int64, ctypes.c_int, ctypes.POINTER(AttnMaskStruct),
                              ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p], ctypes.c_int),
    "ptl_rep_encoder_workspace_size": ([ctypes.c_int64, ctypes.c_int], ctypes.c_size_t),
    "ptl_rep_encoder": ([ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                         ctypes.POINTER(RepWeightsStruct), ctypes.c_void_p, ctypes.c_void_p,
                         ctypes.c_size_t, ctypes.c_void_p], ctypes.c_int),
    "ptl_out_projection": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                            ctypes.c_int, ctypes.POINTER(LayerWeights), ctypes.c_void_p,
                            ctypes.c_size_t, ctypes.c_void_p], ctypes.c_int),
    "ptl_gate": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_int64, ctypes.c_int, ctypes.POINTER(LayerWeights), ctypes.c_void_p,
                  ctypes.c_size_t, ctypes.c_void_p], ctypes.c_int),
    "ptl_route_build": ([ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                         ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p], ctypes.c_int),
    "ptl_moe": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                 ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.POINTER(LayerWeights),
                 ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p], ctypes.c_int),
    "ptl_head": ([ctypes.c_void_p, ctypes.POINTER(HeadWeights), ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t,
                  ctypes.c_void_p], ctypes.c_int),
    "ptl_last_device_error": ([ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p], ctypes.c_int),
    "ptl_wait_selftest": ([ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64,
                           ctypes.c_void_p], ctypes.c_int),
    "ptl_set_trace": ([ctypes.POINTER(Trace)], None),
    "ptl_runner_bucket": ([ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                           ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int32)],
                          ctypes.c_int),
    "ptl_runner_create": ([ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int,
                           ctypes.POINTER(LayerWeights), ctypes.POINTER(HeadWeights), ctypes.c_int32,
                           ctypes.POINTER(ctypes.c_void_p)], ctypes.c_int),
    "ptl_runner_capture": ([ctypes.c_void_p, ctypes.c_int64], ctypes.c_int),
    "ptl_runner_forward": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                            ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                            ctypes.c_void_p, ctypes.c_void_p], ctypes.c_int),
    "ptl_runner_last_device_error": ([ctypes.c_void_p, ctypes.c_void_p], ctypes.c_int),
    "ptl_runner_graphs": ([ctypes.c_void_p], ctypes.c_int32),
    "ptl_runner_destroy": ([ctypes.c_void_p], None),
    "ptl_attention_noalloc": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                               ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p],
                              ctypes.c_int),
    "ptl_quantize_rows_e4m3": ([ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int32,
                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p], ctypes.c_int),
    "ptl_linear_fp8": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                        ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p,
                        ctypes.c_size_t, ctypes.c_void_p], ctypes.c_int),
    "ptl_partition_users": ([ctypes.POINTER(ctypes.c_int32), ctypes.c_int32, ctypes.c_int32,
                             ctypes.POINTER(ctypes.c_int32)], ctypes.c_int),
}


def lib() -> ctypes.CDLL:
    """Load libptl.so (built in-tree by ``packed_sequence_transformer_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m packed_sequence_transformer_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().ptl_status_string(int(s)).decode()


def _check(status: int, where: str):
    if status != 0:
        raise PtlError(status, where)


def _dt(dtype) -> int:
    if dtype in (torch.bfloat16, "bf16", PTL_BF16):
        return PTL_BF16
    if dtype in (torch.float32, "fp32", PTL_F32):
        return PTL_F32
    raise ValueError(f"unsupported dtype {dtype}")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libptl must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def torch_dtype(dt) -> torch.dtype:
    return torch.bfloat16 if _dt(dt) == PTL_BF16 else torch.float32


def layer_struct(w: Dict[str, torch.Tensor]) -> LayerWeights:
    s = LayerWeights()
    for n in LAYER_FIELDS:
        t = w.get(n)
        setattr(s, n, t.data_ptr() if t is not None else None)
    return s


def head_struct(h: Dict[str, torch.Tensor]) -> HeadWeights:
    s = HeadWeights()
    for n in HEAD_FIELDS:
        t = h.get(n)
        setattr(s, n, t.data_ptr() if t is not None else None)
    return s


def to_device_layer(w: Dict, dt, device="cuda") -> Dict[str, torch.Tensor]:
    """numpy/tensor layer parameters -> contiguous device tensors in the ABI's dtypes."""
    tdt = torch_dtype(dt)
    out = {}
    for n in LAYER_FIELDS:
        if n not in w or w[n] is None:
            continue
        t = torch.as_tensor(w[n])
        out[n] = t.to(device=device, dtype=torch.float32 if n in FP32_FIELDS else tdt).contiguous()
    return out


def to_device_head(h: Dict, device="cuda") -> Dict[str, torch.Tensor]:
    return {n: torch.as_tensor(h[n]).to(device=device, dtype=torch.float32).contiguous()
            for n in HEAD_FIELDS if n in h and h[n] is not None}


# ---------------------------------------------------------------- calls
def version() -> int:
    return int(lib().ptl_version())


def workspace_size(max_tokens: int, max_users: int, dtype) -> int:
    return int(lib().ptl_workspace_size(int(max_tokens), int(max_users), _dt(dtype)))


def alloc_workspace(max_tokens: int, max_users: int, dtype, device="cuda") -> torch.Tensor:
    n = workspace_size(max_tokens, max_users, dtype)
    if n == 0:
        raise ValueError("invalid workspace request")
    # zeroed so that the error word reads PTL_OK before any call has used it
    return torch.zeros(n, dtype=torch.uint8, device=device)


def layer_forward(x, out, cu_seqlens, weights, workspace, debug: Optional[Dict] = None, stream=None):
    T = x.shape[0]
    U = cu_seqlens.numel() - 1
    w = layer_struct(weights)
    dbg = None
    if debug:
        dbg = DebugOut(*(debug[k].data_ptr() if debug.get(k) is not None else None
                         for k in ("topk_idx", "topk_w", "perm", "expert_off")))
    _check(lib().ptl_layer_forward(_ptr(x), _ptr(out), _ptr(cu_seqlens), U, T, _dt(x.dtype),
                                   ctypes.byref(w), _ptr(workspace), workspace.numel(),
                                   ctypes.byref(dbg) if dbg is not None else None, _stream(stream)),
           "ptl_layer_forward")
    return out


def stack_forward(x, out, cu_seqlens, layers: List[Dict], workspace, head=None, pred_mask=None,
                  probs=None, n_pred=None, stream=None):
    T = x.shape[0]
    U = cu_seqlens.numel() - 1
    arr = (LayerWeights * len(layers))(*[layer_struct(w) for w in layers])
    hs = head_struct(head) if head is not None else None
    _check(lib().ptl_stack_forward(_ptr(x), _ptr(out), _ptr(cu_seqlens), U, T, len(layers),
                                   _dt(x.dtype), arr, ctypes.byref(hs) if hs is not None else None,
                                   _ptr(pred_mask), _ptr(probs), _ptr(n_pred), _ptr(workspace),
                                   workspace.numel(), _stream(stream)),
           "ptl_stack_forward")
    return out


def qkv_projection(x, qkv, weights, workspace, stream=None):
    w = layer_struct(weights)
    _check(lib().ptl_qkv_projection(_ptr(x), _ptr(qkv), x.shape[0], _dt(x.dtype), ctypes.byref(w),
                                    _ptr(workspace), workspace.numel(), _stream(stream)),
           "ptl_qkv_projection")
    return qkv


def attention(qkv, attn, cu_seqlens, workspace, stream=None):
    _check(lib().ptl_attention(_ptr(qkv), _ptr(attn), _ptr(cu_seqlens), cu_seqlens.numel() - 1,
                               qkv.shape[0], _dt(qkv.dtype), _ptr(workspace), workspace.numel(),
                               _stream(stream)), "ptl_attention")
    return attn


def attention_masked(qkv, attn, cu_seqlens, workspace, causal=True, num_contexts=None,
                     num_targets=None, target_group_size=1, window=0, stream=None):
    """HSTU-style masked attention (``ptl_attention_masked``); num_contexts /
    num_targets: device int32 tensors [U] or None."""
    m = AttnMaskStruct(int(bool(causal)), _ptr(num_contexts), _ptr(num_targets),
                       int(target_group_size), int(window))
    _check(lib().ptl_attention_masked(_ptr(qkv), _ptr(attn), _ptr(cu_seqlens), cu_seqlens.numel() - 1,
                                      qkv.shape[0], _dt(qkv.dtype), ctypes.byref(m), _ptr(workspace),
                                      workspace.numel(), _stream(stream)), "ptl_attention_masked")
    return attn


def rep_encoder_workspace(max_tokens: int, dtype, device="cuda") -> torch.Tensor:
    n = int(lib().ptl_rep_encoder_workspace_size(int(max_tokens), _dt(dtype)))
    if n == 0:
        raise ValueError("invalid RepEncoder workspace request")
    return torch.empty(n, dtype=torch.uint8, device=device)


def rep_weights_struct(tables, ln_g, ln_b, w, b=None) -> RepWeightsStruct:
    """28 device tables [vocab_s, 512] (dt), LN params [14336] (f32), W [512, 14336] (dt), b [512] (f32)."""
    if len(tables) != 28:
        raise ValueError("the RepEncoder has 28 slots")
    st = RepWeightsStruct()
    for i, t in enumerate(tables):
        st.tables[i] = t.data_ptr() if t.numel() else 0
        st.vocab[i] = t.shape[0]
    st.ln_g, st.ln_b, st.w = ln_g.data_ptr(), ln_b.data_ptr(), w.data_ptr()
    st.b = b.data_ptr() if b is not None else None
    return st


def rep_encoder(ids, bag_offsets, num_tokens, weights: RepWeightsStruct, out, workspace, stream=None):
    """RepEncoder front end (``ptl_rep_encoder``): embedding bags, LayerNorm
    over 14336, Linear to 512 into out [T, 512] (dt of out)."""
    _check(lib().ptl_rep_encoder(_ptr(ids), ids.numel(), _ptr(bag_offsets), int(num_tokens), _dt(out.dtype),
                                 ctypes.byref(weights), _ptr(out), _ptr(workspace), workspace.numel(),
                                 _stream(stream)), "ptl_rep_encoder")
    return out


def out_projection(attn, x, x1, weights, workspace, stream=None):
    w = layer_struct(weights)
    _check(lib().ptl_out_projection(_ptr(attn), _ptr(x), _ptr(x1), x.shape[0], _dt(x.dtype),
                                    ctypes.byref(w), _ptr(workspace), workspace.numel(),
                                    _stream(stream)), "ptl_out_projection")
    return x1


def gate(x1, xn2, topk_idx, topk_w, weights, workspace, stream=None):
    w = layer_struct(weights)
    _check(lib().ptl_gate(_ptr(x1), _ptr(xn2), _ptr(topk_idx), _ptr(topk_w), x1.shape[0],
                          _dt(xn2.dtype), ctypes.byref(w), _ptr(workspace), workspace.numel(),
                          _stream(stream)), "ptl_gate")
    return xn2, topk_idx, topk_w


def route_build(topk_idx, perm, expert_off, workspace, stream=None):
    _check(lib().ptl_route_build(_ptr(topk_idx), topk_idx.shape[0], _ptr(perm), _ptr(expert_off),
                                 _ptr(workspace), workspace.numel(), _stream(stream)),
           "ptl_route_build")
    return perm, expert_off


def moe(xn2, topk_idx, topk_w, residual, out, weights, workspace, stream=None):
    w = layer_struct(weights)
    _check(lib().ptl_moe(_ptr(xn2), _ptr(topk_idx), _ptr(topk_w), _ptr(residual), _ptr(out),
                         xn2.shape[0], _dt(xn2.dtype), ctypes.byref(w), _ptr(workspace),
                         workspace.numel(), _stream(stream)), "ptl_moe")
    return out


def head(h, head_weights, pred_mask, probs, n_pred, workspace, stream=None):
    hs = head_struct(head_weights)
    _check(lib().ptl_head(_ptr(h), ctypes.byref(hs), _ptr(pred_mask), _ptr(probs), _ptr(n_pred),
                          h.shape[0], _dt(h.dtype), _ptr(workspace), workspace.numel(),
                          _stream(stream)), "ptl_head")
    return probs


def attention_noalloc(qkv, attn, cu_seqlens, device_status=None, stream=None):
    """ptl_attention_noalloc: the attention step for callers that cannot
    allocate device memory (no workspace; scratch in a fixed array inside the
    library).  device_status, if given, is a device int32 tensor that
    receives the call's device-side status."""
    _check(lib().ptl_attention_noalloc(_ptr(qkv), _ptr(attn), _ptr(cu_seqlens),
                                       cu_seqlens.numel() - 1, qkv.shape[0], _dt(qkv.dtype),
                                       _ptr(device_status), _stream(stream)),
           "ptl_attention_noalloc")
    return attn


def quantize_rows_e4m3(x, codes=None, scales=None, stream=None):
    """ptl_quantize_rows_e4m3: per-row e4m3 codes (uint8 tensor) and float32
    scales of a 2-D bf16 / fp32 device tensor."""
    rows, cols = x.shape
    codes = codes if codes is not None else torch.empty(rows, cols, dtype=torch.uint8, device=x.device)
    scales = scales if scales is not None else torch.empty(rows, dtype=torch.float32, device=x.device)
    _check(lib().ptl_quantize_rows_e4m3(_ptr(x), _dt(x.dtype), rows, cols, _ptr(codes), _ptr(scales),
                                        _stream(stream)), "ptl_quantize_rows_e4m3")
    return codes, scales


def linear_fp8(xq, sx, wq, sw, bias, out, workspace, stream=None):
    """ptl_linear_fp8: out (bf16 [M][N]) = (xq wq^T) * sx[m] * sw[n] + bias[n]."""
    M, K = xq.shape
    N = wq.shape[0]
    _check(lib().ptl_linear_fp8(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), _ptr(bias), _ptr(out), M, K, N,
                                _ptr(workspace), workspace.numel(), _stream(stream)), "ptl_linear_fp8")
    return out


def partition_users(cu_seqlens, num_parts: int):
    """ptl_partition_users: contiguous user ranges, one per part, balanced by
    cost (host offsets in, host int32 [num_parts + 1] user boundaries out)."""
    import numpy as np
    cu = np.ascontiguousarray(np.asarray(cu_seqlens), dtype=np.int32)
    begin = np.zeros(num_parts + 1, dtype=np.int32)
    _check(lib().ptl_partition_users(cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), cu.size - 1,
                                     num_parts, begin.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))),
           "ptl_partition_users")
    return begin


def part_of_batch(cu_seqlens, user_begin, part: int):
    """The slice of a batch that part `part` runs: (first token, end token,
    first user, end user, rebased offsets int32 [users + 1])."""
    import numpy as np
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    b, e = int(user_begin[part]), int(user_begin[part + 1])
    t0, t1 = int(cu[b]), int(cu[e])
    return t0, t1, b, e, (cu[b:e + 1] - t0).astype(np.int32)


def last_device_error(workspace, stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device error word."""
    return int(lib().ptl_last_device_error(_ptr(workspace), workspace.numel(), _stream(stream)))


def runner_bucket(total_tokens: int, max_users: int, stride: int = 0):
    """(bucket tokens, padded user count) a runner uses for a batch of
    ``total_tokens`` (host arithmetic only)."""
    b, u = ctypes.c_int64(), ctypes.c_int32()
    _check(lib().ptl_runner_bucket(int(total_tokens), int(max_users), int(stride), ctypes.byref(b),
                                   ctypes.byref(u)), "ptl_runner_bucket")
    return b.value, u.value


class StackRunner:
    """The layer stack (and optional head) as one CUDA graph per token
    bucket (``ptl_runner_*``): inputs and outputs may be host (ideally
    pinned) or device tensors; calls must be ordered on one stream."""

    def __init__(self, max_tokens: int, max_users: int, layers: List[Dict], dtype, head=None,
                 stride: int = 0):
        self._keep = (layers, head)  # the device weights must outlive the runner
        arr = (LayerWeights * len(layers))(*[layer_struct(w) for w in layers])
        hs = head_struct(head) if head is not None else None
        r = ctypes.c_void_p()
        _check(lib().ptl_runner_create(int(max_tokens), int(max_users), len(layers), _dt(dtype), arr,
                                       ctypes.byref(hs) if hs is not None else None, int(stride),
                                       ctypes.byref(r)), "ptl_runner_create")
        self._r = r
        self.has_head = head is not None

    def capture(self, total_tokens: int) -> None:
        _check(lib().ptl_runner_capture(self._r, int(total_tokens)), "ptl_runner_capture")

    def forward(self, x, cu_seqlens, out=None, pred_mask=None, probs=None, n_pred=None,
                stream=None):
        _check(lib().ptl_runner_forward(self._r, _ptr(x), _ptr(out), _ptr(cu_seqlens),
                                        cu_seqlens.numel() - 1, x.shape[0], _ptr(pred_mask),
                                        _ptr(probs), _ptr(n_pred), _stream(stream)),
               "ptl_runner_forward")
        return out

    def last_device_error(self, stream=None) -> int:
        return int(lib().ptl_runner_last_device_error(self._r, _stream(stream)))

    def graphs(self) -> int:
        return int(lib().ptl_runner_graphs(self._r))

    def close(self) -> None:
        if getattr(self, "_r", None):
            lib().ptl_runner_destroy(self._r)
            self._r = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def wait_selftest(workspace, which: int, limit_ns: int, stream=None) -> None:
    """Launches a kernel whose bounded wait (0: mbarrier, 1: global flag) runs
    out after ``limit_ns``; ``last_device_error`` then reports PTL_ERR_TIMEOUT."""
    _check(lib().ptl_wait_selftest(_ptr(workspace), workspace.numel(), int(which), int(limit_ns),
                                   _stream(stream)), "ptl_wait_selftest")


class KernelTrace:
    """Context manager recording a CUDA event before every kernel the library
    enqueues from this thread (and one after the last), so the device time
    of each launch can be read afterwards with ``launches()``."""

    def __init__(self, capacity: int = 4096):
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(capacity)]
        s = torch.cuda.current_stream()
        for e in self.events:  # torch creates the CUDA event at its first record
            e.record(s)
        torch.cuda.synchronize()
        self._handles = (ctypes.c_void_p * capacity)(*[e.cuda_event for e in self.events])
        self._kinds = (ctypes.c_int32 * capacity)()
        self.trace = Trace(self._handles, self._kinds, capacity, 0)

    def __enter__(self):
        self.trace.count = 0
        lib().ptl_set_trace(ctypes.byref(self.trace))
        return self

    def __exit__(self, *exc):
        lib().ptl_set_trace(None)
        return False

    def launches(self):
        """[(kind name, milliseconds)] for each recorded launch (synchronises)."""
        torch.cuda.synchronize()
        out = []
        n = self.trace.count
        for i in range(n - 1):
            k = self._kinds[i]
            if k == 99:
                continue
            out.append((KERNEL_KINDS.get(k, str(k)), self.events[i].elapsed_time(self.events[i + 1])))
        return out
