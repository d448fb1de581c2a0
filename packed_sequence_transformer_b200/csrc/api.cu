// api.cu -- the C ABI of libptl: argument validation, workspace carving,
// TMA descriptor encoding and the launch sequence of the layer, the stack
// and the individual steps.  No allocation, no stream synchronisation (except
// in ptl_last_device_error), no state kept between calls.
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "../../include/ptl.h"
#include "common.cuh"
#include "launch.h"

namespace ptl {

thread_local ptl_trace* g_trace = nullptr;

// NVTX annotations (NVTX3, header-only: each call is a no-op unless a
// profiler is attached).  Every entry point opens a range named after itself
// and, nested in it, one range per kernel launch named by the launch's kind,
// so a profiler can attribute and filter the library's kernels; the
// entry point's guard closes both on every return path.
static const char* kind_name(int kind) {
  switch (kind) {
    case PTL_KERNEL_CLEAR: return "clear";
    case PTL_KERNEL_WORKLIST: return "worklist";
    case PTL_KERNEL_LAYERNORM: return "layernorm";
    case PTL_KERNEL_GEMM_QKV: return "gemm_qkv";
    case PTL_KERNEL_ATTENTION: return "attention";
    case PTL_KERNEL_GEMM_OUT: return "gemm_out";
    case PTL_KERNEL_GATE: return "gate";
    case PTL_KERNEL_ROUTE: return "route";
    case PTL_KERNEL_GEMM_EXPERT1: return "gemm_expert1";
    case PTL_KERNEL_GEMM_EXPERT2: return "gemm_expert2";
    case PTL_KERNEL_HEAD: return "head";
    case PTL_KERNEL_COPY: return "copy";
    case PTL_KERNEL_COMBINE: return "combine";
    default: return "ptl";
  }
}
static thread_local bool g_nvtx_kernel_open = false;
static void nvtx_kernel(int kind) {
  if (kind == PTL_KERNEL_END) return;
  if (g_nvtx_kernel_open) nvtxRangePop();
  nvtxRangePushA(kind_name(kind));
  g_nvtx_kernel_open = true;
}
void api_range_push(const char* name) { nvtxRangePushA(name); }
void api_range_pop() {
  if (g_nvtx_kernel_open) nvtxRangePop();
  g_nvtx_kernel_open = false;
  nvtxRangePop();
}

void trace_mark(cudaStream_t st, int kind) {
  nvtx_kernel(kind);
  ptl_trace* t = g_trace;
  if (!t || !t->events || t->count >= t->capacity) return;
  // inside a stream capture only an external record becomes an event node
  // that can be timed after the graph runs
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(st, &cap);
  if (cap == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(static_cast<cudaEvent_t>(t->events[t->count]), st, cudaEventRecordExternal);
  else
    cudaEventRecord(static_cast<cudaEvent_t>(t->events[t->count]), st);
  if (t->kinds) t->kinds[t->count] = kind;
  ++t->count;
}

}  // namespace ptl

namespace {
using namespace ptl;

// ------------------------------------------------------------ driver entry
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2D bf16 tensor map: `rows` rows of `cols` elements, `stride_bytes` apart;
// box = box_rows x box_cols (box_cols * 2 bytes = 128, the swizzle span).
bool map_bf16(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t stride_bytes,
              uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {stride_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D fp32 tensor map, box = box_rows x box_cols (box_cols * 4 bytes = 128).
bool map_f32(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t stride_bytes,
             uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {stride_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D byte tensor map (e4m3 codes): box = box_rows x 128 bytes (the swizzle span).
bool map_u8(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t stride_bytes,
            uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {stride_bytes};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

ptl_status device_ok() {
  static int cache[64];  // 0 unknown, 1 ok, 2 unsupported
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PTL_ERR_CUDA;
  if (dev >= 0 && dev < 64 && cache[dev]) return cache[dev] == 1 ? PTL_OK : PTL_ERR_UNSUPPORTED;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return PTL_ERR_CUDA;
  const int ok = major == 10 ? 1 : 2;
  if (dev >= 0 && dev < 64) cache[dev] = ok;
  return ok == 1 ? PTL_OK : PTL_ERR_UNSUPPORTED;
}

inline bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool a4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
inline bool a8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }
inline bool opt16(const void* p) { return p == nullptr || a16(p); }

ptl_status check_common(int64_t T, ptl_dtype dt, void* ws, size_t ws_bytes, int32_t U, WsLayout* L) {
  if (dt != PTL_F32 && dt != PTL_BF16) return PTL_ERR_DTYPE;
  if (T < 0 || T >= (int64_t(1) << 31) || U < 1) return PTL_ERR_SHAPE;
  if (!ws) return PTL_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return PTL_ERR_ALIGN;
  if (!make_layout(T, U, dt, L)) return PTL_ERR_SHAPE;
  if (ws_bytes < L->total) return PTL_ERR_WORKSPACE;
  return PTL_OK;
}

ptl_status check_weights(const ptl_layer_weights* w) {
  if (!w) return PTL_ERR_NULL;
  const void* req[] = {w->ln1_g, w->ln1_b, w->w_qkv, w->w_o, w->ln2_g, w->ln2_b, w->w_gate, w->w1, w->w2};
  for (const void* p : req) {
    if (!p) return PTL_ERR_NULL;
    if (!a16(p)) return PTL_ERR_ALIGN;
  }
  const void* opt[] = {w->b_qkv, w->b_o, w->b_gate, w->b1, w->b2};
  for (const void* p : opt)
    if (!opt16(p)) return PTL_ERR_ALIGN;
  return PTL_OK;
}

ptl_status check_head(const ptl_head_weights* h) {
  if (!h->lnf_g || !h->lnf_b || !h->w) return PTL_ERR_NULL;
  if (!a16(h->lnf_g) || !a16(h->lnf_b) || !a16(h->w) || !opt16(h->b)) return PTL_ERR_ALIGN;
  return PTL_OK;
}

inline void mark(cudaStream_t st, int kind) { trace_mark(st, kind); }

struct Call {
  WsLayout L;
  char* ws;
  int32_t* err;
  cudaStream_t st;
  ptl_dtype dt;
  int T;
  int U;
};

inline const float* F32(const void* p) { return static_cast<const float*>(p); }
template <typename T>
inline T* at(const Call& c, size_t off) { return reinterpret_cast<T*>(c.ws + off); }

#define PTL_TRY(expr)                 \
  do {                                \
    if ((expr) != 0) return PTL_ERR_CUDA; \
  } while (0)

// Clears the error word (every top-level call reports only its own errors)
// and the routing state the gate starts from (per-chunk expert counts, the
// fused gate + route look-back state; the first expert GEMM of each layer
// clears them again once they are used).  The work list in between is
// rewritten by the work-list kernel.
ptl_status begin(const Call& c) {
  mark(c.st, PTL_KERNEL_CLEAR);
  return cudaMemsetAsync(c.ws, 0, c.L.clear_end, c.st) == cudaSuccess ? PTL_OK : PTL_ERR_CUDA;
}

// xn_ready: LayerNorm1 of x is already in the workspace (the previous
// layer's combine wrote it).
ptl_status step_qkv(const Call& c, const void* x, void* qkv, const ptl_layer_weights* w,
                    bool xn_ready = false) {
  const int T = c.T;
  if (c.dt == PTL_BF16) {
    if (!xn_ready) {
      mark(c.st, PTL_KERNEL_LAYERNORM);
      PTL_TRY(launch_layernorm(x, F32(w->ln1_g), F32(w->ln1_b), c.ws + c.L.xn, T, c.dt, c.st));
    }
    CUtensorMap ma, mb, mo;
    if (!map_bf16(&ma, c.ws + c.L.xn, D, T, D * 2, 64, 128)) return PTL_ERR_CUDA;
    if (!map_bf16(&mb, w->w_qkv, D, QKV_N, D * 2, 64, QKV_BN / 2)) return PTL_ERR_CUDA;
    if (!map_bf16(&mo, qkv, QKV_N, T, QKV_N * 2, 64, 128)) return PTL_ERR_CUDA;
    mark(c.st, PTL_KERNEL_GEMM_QKV);
    // the expert weights (16 MB, read once per layer) start coming into L2
    // while the attention and the gate run, which leave HBM mostly idle
    const size_t expert_w_bytes = size_t(E) * F * D * 2;
    PTL_TRY(launch_gemm_qkv(ma, mb, mo, F32(w->b_qkv), qkv, T, c.err, c.st, w->w1, expert_w_bytes, w->w2,
                            expert_w_bytes));
  } else {
    mark(c.st, PTL_KERNEL_LAYERNORM);
    PTL_TRY(launch_layernorm(x, F32(w->ln1_g), F32(w->ln1_b), c.ws + c.L.xn, T, c.dt, c.st));
    mark(c.st, PTL_KERNEL_GEMM_QKV);
    PTL_TRY(launch_gemm_f32(0, at<float>(c, c.L.xn), D, F32(w->w_qkv), F32(w->b_qkv), nullptr,
                            static_cast<float*>(qkv), QKV_N, T, QKV_N, D, c.L, c.ws, c.st));
  }
  return PTL_OK;
}

// list_early: a kernel (the QKV projection) runs between the work list and
// the attention
ptl_status step_attention(const Call& c, const void* qkv, void* attn, const int32_t* cu,
                          const AttnMask* mask = nullptr, bool list_early = false) {
  if (c.dt == PTL_BF16) {
    CUtensorMap m;
    if (!map_bf16(&m, qkv, QKV_N, c.T, QKV_N * 2, 64, 128)) return PTL_ERR_CUDA;
    mark(c.st, PTL_KERNEL_ATTENTION);
    PTL_TRY(launch_attn_tc(m, attn, cu, c.L, c.ws, c.st, mask, list_early));
  } else {
    mark(c.st, PTL_KERNEL_ATTENTION);
    PTL_TRY(launch_attn_f32(static_cast<const float*>(qkv), static_cast<float*>(attn), cu, c.L, c.ws,
                            c.st, mask));
  }
  return PTL_OK;
}

ptl_status step_out(const Call& c, const void* attn, const void* x, void* x1, const ptl_layer_weights* w) {
  if (c.dt == PTL_BF16) {
    CUtensorMap ma, mb, mo;
    if (!map_bf16(&ma, attn, D, c.T, D * 2, 64, 128)) return PTL_ERR_CUDA;
    if (!map_bf16(&mb, w->w_o, D, D, D * 2, 64, OUT_BN / 2)) return PTL_ERR_CUDA;
    if (!map_f32(&mo, x1, D, c.T, D * 4, 32, 128)) return PTL_ERR_CUDA;
    mark(c.st, PTL_KERNEL_GEMM_OUT);
    PTL_TRY(launch_gemm_out(ma, mb, mo, F32(w->b_o), x, x1, c.T, c.err, c.st));
  } else {
    mark(c.st, PTL_KERNEL_GEMM_OUT);
    PTL_TRY(launch_gemm_f32(1, static_cast<const float*>(attn), D, F32(w->w_o), F32(w->b_o),
                            static_cast<const float*>(x), static_cast<float*>(x1), D, c.T, D, D, c.L,
                            c.ws, c.st));
  }
  return PTL_OK;
}

ptl_status step_gate(const Call& c, const void* x1, void* xn2, int32_t* idx, float* wout,
                     const ptl_layer_weights* w) {
  mark(c.st, PTL_KERNEL_GATE);
  PTL_TRY(launch_gate(x1, F32(w->ln2_g), F32(w->ln2_b), F32(w->w_gate), F32(w->b_gate), xn2, idx, wout,
                      at<int32_t>(c, c.L.chunk_cnt), c.T, c.dt, c.st));
  return PTL_OK;
}

// Routes + both expert GEMMs + combine + residual.  The per-chunk expert
// counts must already be in the workspace.
ptl_status step_experts(const Call& c, const float* wts, const void* resid, void* out,
                        const ptl_layer_weights* w, const ptl_layer_weights* next, bool fused = false,
                        const HeadArgs* head = nullptr);

// next (bf16 build, nullable): the following layer, whose LayerNorm1 of `out`
// the combine also writes into the workspace.
ptl_status step_moe(const Call& c, const void* xn2, const int32_t* idx, const float* wts,
                    const void* resid, void* out, const ptl_layer_weights* w, int32_t* dbg_perm,
                    int32_t* dbg_off, const ptl_layer_weights* next = nullptr) {
  mark(c.st, PTL_KERNEL_ROUTE);
  PTL_TRY(launch_route(idx, c.T, c.L, c.ws, dbg_perm, dbg_off, c.dt == PTL_BF16 ? xn2 : nullptr, c.st));
  if (c.dt == PTL_BF16) return step_experts(c, wts, resid, out, w, next);
  // the route builder has consumed the per-chunk expert counts: clear them
  // for the next gate (the bf16 path's first expert GEMM does this)
  if (cudaMemsetAsync(c.ws + c.L.chunk_cnt, 0, sizeof(int32_t) * size_t(c.L.n_chunks) * E, c.st) != cudaSuccess)
    return PTL_ERR_CUDA;
  mark(c.st, PTL_KERNEL_GEMM_EXPERT1);
  PTL_TRY(launch_gemm_f32(2, static_cast<const float*>(xn2), D, F32(w->w1), F32(w->b1), nullptr,
                          at<float>(c, c.L.hbuf), F, 0, F, D, c.L, c.ws, c.st));
  mark(c.st, PTL_KERNEL_GEMM_EXPERT2);
  PTL_TRY(launch_gemm_f32(3, at<float>(c, c.L.hbuf), F, F32(w->w2), F32(w->b2), nullptr,
                          at<float>(c, c.L.ybuf), D, 0, D, F, c.L, c.ws, c.st));
  mark(c.st, PTL_KERNEL_COMBINE);
  PTL_TRY(launch_combine_f32(at<float>(c, c.L.ybuf), wts, static_cast<const float*>(resid),
                             static_cast<float*>(out), c.T, c.err, c.st));
  return PTL_OK;
}

// bf16: both expert GEMMs over the routed rows already in the workspace
// (xperm, tiles, meta, pos), then the combine + residual (+ the next layer's
// LayerNorm1 inside a stack).
// fused: both expert GEMMs in one launch (the layer path, whose gate +
// route kernel cleared the per-tile counters).  head (nullable): the last
// layer of a bf16 stack, whose combine also computes the prediction head.
ptl_status step_experts(const Call& c, const float* wts, const void* resid, void* out,
                        const ptl_layer_weights* w, const ptl_layer_weights* next, bool fused,
                        const HeadArgs* head) {
  {
    CUtensorMap mx, m1, m2, mh, my;
    if (!map_bf16(&mx, c.ws + c.L.xperm, D, c.L.padded_rows, D * 2, 64, 128)) return PTL_ERR_CUDA;
    if (!map_bf16(&m1, w->w1, D, uint64_t(E) * F, D * 2, 64, MOE1_BN / 2)) return PTL_ERR_CUDA;
    if (!map_bf16(&m2, w->w2, F, uint64_t(E) * D, F * 2, 64, GEMM2_BN / 2)) return PTL_ERR_CUDA;
    if (!map_bf16(&mh, c.ws + c.L.hbuf, F, c.L.padded_rows, F * 2, 64, 128)) return PTL_ERR_CUDA;
    if (!map_bf16(&my, c.ws + c.L.ybuf, D, c.L.padded_rows, D * 2, 64, 128)) return PTL_ERR_CUDA;
    if (fused) {
      mark(c.st, PTL_KERNEL_GEMM_EXPERT1);
      PTL_TRY(launch_gemm_moe12(mx, m1, mh, m2, my, F32(w->b1), F32(w->b2), c.L, c.ws, c.st));
    } else {
      mark(c.st, PTL_KERNEL_GEMM_EXPERT1);
      PTL_TRY(launch_gemm_moe1(mx, m1, mh, F32(w->b1), c.L, c.ws, c.st));
      mark(c.st, PTL_KERNEL_GEMM_EXPERT2);
      PTL_TRY(launch_gemm_moe2(mh, m2, my, F32(w->b2), c.L, c.ws, c.st));
    }
    mark(c.st, PTL_KERNEL_COMBINE);
    // after the fused launch, when the combine's blocks fit one wave at 8 per
    // SM (its waiting blocks then stay few beside the expert launch), the
    // combine starts on the finished tiles instead of waiting for the launch
    const bool streamed = fused && (c.T + 7) / 8 <= 8 * num_sms();
    PTL_TRY(launch_combine_bf16(c.ws + c.L.ybuf, at<int32_t>(c, c.L.pos), wts,
                                static_cast<const float*>(resid), out, c.T,
                                next ? F32(next->ln1_g) : nullptr, next ? F32(next->ln1_b) : nullptr,
                                next ? c.ws + c.L.xn : nullptr, c.err, c.st, streamed ? &c.L : nullptr, c.ws,
                                head));
  }
  return PTL_OK;
}

// xn_ready: LayerNorm1 of x is already in the workspace; next (nullable,
// bf16 build): the following layer of a stack, whose LayerNorm1 the combine
// computes on the way out; head (nullable, bf16 build): the prediction head,
// computed by the combine of the stack's last layer.
ptl_status layer_body(const Call& c, const void* x, void* out, const int32_t* cu,
                      const ptl_layer_weights* w, const ptl_debug_out* dbg, bool xn_ready = false,
                      const ptl_layer_weights* next = nullptr, const HeadArgs* head = nullptr) {
  ptl_status s;
  if ((s = step_qkv(c, x, c.ws + c.L.qkv, w, xn_ready)) != PTL_OK) return s;
  if ((s = step_attention(c, c.ws + c.L.qkv, c.ws + c.L.attn, cu, nullptr, true)) != PTL_OK) return s;
  if ((s = step_out(c, c.ws + c.L.attn, x, c.ws + c.L.x1, w)) != PTL_OK) return s;
  int32_t* idx = at<int32_t>(c, c.L.idx);
  float* wts = at<float>(c, c.L.wgt);
  if (c.dt == PTL_BF16) {
    // gate + route builder in one kernel, then the experts and the combine
    mark(c.st, PTL_KERNEL_GATE);
    PTL_TRY(launch_gate_route(c.ws + c.L.x1, F32(w->ln2_g), F32(w->ln2_b), F32(w->w_gate), F32(w->b_gate), c.T,
                              c.L, c.ws, c.st));
    if (dbg && (dbg->perm || dbg->expert_off)) {
      mark(c.st, PTL_KERNEL_ROUTE);
      PTL_TRY(launch_route_debug(c.T, c.L, c.ws, dbg->perm, dbg->expert_off, c.st));
    }
    if ((s = step_experts(c, wts, c.ws + c.L.x1, out, w, next, true, head)) != PTL_OK) return s;
  } else {
    if ((s = step_gate(c, c.ws + c.L.x1, c.ws + c.L.xn2, idx, wts, w)) != PTL_OK) return s;
    if ((s = step_moe(c, c.ws + c.L.xn2, idx, wts, c.ws + c.L.x1, out, w, dbg ? dbg->perm : nullptr,
                      dbg ? dbg->expert_off : nullptr, next)) != PTL_OK)
      return s;
  }
  if (dbg && (dbg->topk_idx || dbg->topk_w)) mark(c.st, PTL_KERNEL_COPY);
  if (dbg && dbg->topk_idx &&
      cudaMemcpyAsync(dbg->topk_idx, idx, sizeof(int32_t) * 2 * c.T, cudaMemcpyDeviceToDevice, c.st) !=
          cudaSuccess)
    return PTL_ERR_CUDA;
  if (dbg && dbg->topk_w &&
      cudaMemcpyAsync(dbg->topk_w, wts, sizeof(float) * 2 * c.T, cudaMemcpyDeviceToDevice, c.st) !=
          cudaSuccess)
    return PTL_ERR_CUDA;
  return PTL_OK;
}

ptl_status setup(Call* c, int64_t T, int32_t U, ptl_dtype dt, void* ws, size_t ws_bytes, void* stream) {
  ptl_status s = check_common(T, dt, ws, ws_bytes, U, &c->L);
  if (s != PTL_OK) return s;
  c->ws = static_cast<char*>(ws);
  c->err = reinterpret_cast<int32_t*>(c->ws + c->L.err);
  c->st = static_cast<cudaStream_t>(stream);
  c->dt = dt;
  c->T = int(T);
  c->U = U;
  return PTL_OK;
}

}  // namespace

extern "C" {

int32_t ptl_version(void) { return PTL_VERSION; }

void ptl_set_trace(ptl_trace* trace) { ptl::g_trace = trace; }

const char* ptl_status_string(ptl_status s) {
  switch (s) {
    case PTL_OK: return "ok";
    case PTL_ERR_NULL: return "a required pointer is NULL";
    case PTL_ERR_ALIGN: return "a pointer is not aligned (16 bytes; workspace 256 bytes)";
    case PTL_ERR_SHAPE: return "invalid size or index (num_users < 1, total_tokens out of [0, 2^31), expert id out of range)";
    case PTL_ERR_BAD_OFFSETS: return "cu_seqlens is not 0-based, non-decreasing and ending at total_tokens";
    case PTL_ERR_WORKSPACE: return "workspace smaller than ptl_workspace_size()";
    case PTL_ERR_DTYPE: return "unknown dtype";
    case PTL_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
    case PTL_ERR_TIMEOUT: return "a bounded device-side wait ran out";
    case PTL_ERR_BAD_IDS: return "an embedding id outside its table, or bag offsets not within 0 .. num_ids and non-decreasing";
    case PTL_ERR_BAD_MASK: return "attention mask: target_group_size < 1, causal not 0/1, or a user's contextual + candidate counts outside 0 .. its length";
    case PTL_ERR_UNSUPPORTED: return "unsupported device (needs sm_100)";
  }
  return "unknown status";
}

size_t ptl_workspace_size(int64_t max_tokens, int32_t max_users, ptl_dtype dt) {
  WsLayout L;
  if (!make_layout(max_tokens, max_users, dt, &L)) return 0;
  return L.total;
}

ptl_status ptl_layer_forward(const void* x, void* out, const int32_t* cu_seqlens, int32_t num_users,
                             int64_t total_tokens, ptl_dtype dt, const ptl_layer_weights* w,
                             void* workspace, size_t ws_bytes, const ptl_debug_out* dbg, void* stream) {
  ApiRange nvtx_range{"ptl_layer_forward"};
  Call c;
  ptl_status s = setup(&c, total_tokens, num_users, dt, workspace, ws_bytes, stream);
  if (s != PTL_OK) return s;
  if (total_tokens == 0) return PTL_OK;
  if (!x || !out || !cu_seqlens) return PTL_ERR_NULL;
  if (!a16(x) || !a16(out) || !a4(cu_seqlens)) return PTL_ERR_ALIGN;
  if ((s = check_weights(w)) != PTL_OK) return s;
  if (x == out) return PTL_ERR_SHAPE;
  if ((s = device_ok()) != PTL_OK) return s;
  if ((s = begin(c)) != PTL_OK) return s;
  EndMark end_mark{c.st};
  mark(c.st, PTL_KERNEL_WORKLIST);
  if (c.dt == PTL_BF16) {
    // the work list and LayerNorm1 of x in one launch
    PTL_TRY(launch_prologue(cu_seqlens, num_users, c.T, c.L, c.ws, x, F32(w->ln1_g), F32(w->ln1_b), c.ws + c.L.xn,
                            c.st));
    return layer_body(c, x, out, cu_seqlens, w, dbg, true);
  }
  PTL_TRY(launch_worklist(cu_seqlens, num_users, c.T, c.L, c.ws, c.st));
  return layer_body(c, x, out, cu_seqlens, w, dbg);
}

ptl_status ptl_stack_forward(const void* x, void* out, const int32_t* cu_seqlens, int32_t num_users,
                             int64_t total_tokens, int32_t num_layers, ptl_dtype dt,
                             const ptl_layer_weights* layers, const ptl_head_weights* head,
                             const uint8_t* pred_mask, float* probs, int32_t* n_pred, void* workspace,
                             size_t ws_bytes, void* stream) {
  ApiRange nvtx_range{"ptl_stack_forward"};
  Call c;
  ptl_status s = setup(&c, total_tokens, num_users, dt, workspace, ws_bytes, stream);
  if (s != PTL_OK) return s;
  if (total_tokens == 0) return PTL_OK;
  if (num_layers < 1) return PTL_ERR_SHAPE;
  if (!x || !out || !cu_seqlens || !layers) return PTL_ERR_NULL;
  if (!a16(x) || !a16(out) || !a4(cu_seqlens)) return PTL_ERR_ALIGN;
  if (x == out) return PTL_ERR_SHAPE;
  for (int i = 0; i < num_layers; ++i)
    if ((s = check_weights(&layers[i])) != PTL_OK) return s;
  if (head) {
    if ((s = check_head(head)) != PTL_OK) return s;
    if (!pred_mask || !probs) return PTL_ERR_NULL;
    if (!a4(probs) || (n_pred && !a4(n_pred))) return PTL_ERR_ALIGN;
  }
  if ((s = device_ok()) != PTL_OK) return s;
  if ((s = begin(c)) != PTL_OK) return s;
  EndMark end_mark{c.st};
  mark(c.st, PTL_KERNEL_WORKLIST);
  const bool fuse = c.dt == PTL_BF16;
  if (fuse) {
    // the work list and layer 0's LayerNorm1 of x in one launch
    // (with a head, also the head's output slots from the prediction mask)
    PTL_TRY(launch_prologue(cu_seqlens, num_users, c.T, c.L, c.ws, x, F32(layers[0].ln1_g), F32(layers[0].ln1_b),
                            c.ws + c.L.xn, c.st, head ? pred_mask : nullptr, head ? n_pred : nullptr));
  } else {
    PTL_TRY(launch_worklist(cu_seqlens, num_users, c.T, c.L, c.ws, c.st));
  }
  const void* h_in = x;
  for (int i = 0; i < num_layers; ++i) {
    void* h_out = (i == num_layers - 1) ? out : c.ws + ((i & 1) ? c.L.act1 : c.L.act0);
    // bf16: layer i's combine also writes LayerNorm1 of its output for layer
    // i + 1 (layer 0's comes from the prologue)
    const ptl_layer_weights* next = (fuse && i + 1 < num_layers) ? &layers[i + 1] : nullptr;
    // bf16 with a head: the last layer's combine computes it, each kept
    // token's probability going to the slot the prologue gave it
    const HeadArgs hd{head ? F32(head->lnf_g) : nullptr, head ? F32(head->lnf_b) : nullptr,
                      head ? F32(head->w) : nullptr, head ? F32(head->b) : nullptr, probs,
                      reinterpret_cast<const int32_t*>(c.ws + c.L.head_p)};
    const bool head_here = fuse && head && i == num_layers - 1;
    if ((s = layer_body(c, h_in, h_out, cu_seqlens, &layers[i], nullptr, fuse, next, head_here ? &hd : nullptr)) !=
        PTL_OK)
      return s;
    h_in = h_out;
  }
  if (head && !fuse) {
    mark(c.st, PTL_KERNEL_HEAD);
    PTL_TRY(launch_head(out, head, pred_mask, probs, n_pred, c.T, c.dt, c.L, c.ws, c.st));
  }
  return PTL_OK;
}

ptl_status ptl_qkv_projection(const void* x, void* qkv, int64_t total_tokens, ptl_dtype dt,
                              const ptl_layer_weights* w, void* workspace, size_t ws_bytes, void* stream) {
  ApiRange nvtx_range{"ptl_qkv_projection"};
  Call c;
  ptl_status s = setup(&c, total_tokens, 1, dt, workspace, ws_bytes, stream);
  if (s != PTL_OK) return s;
  if (total_tokens == 0) return PTL_OK;
  if (!x || !qkv || !w || !w->ln1_g || !w->ln1_b || !w->w_qkv) return PTL_ERR_NULL;
  if (!a16(x) || !a16(qkv) || !a16(w->ln1_g) || !a16(w->ln1_b) || !a16(w->w_qkv) || !opt16(w->b_qkv))
    return PTL_ERR_ALIGN;
  if ((s = device_ok()) != PTL_OK) return s;
  if ((s = begin(c)) != PTL_OK) return s;
  EndMark end_mark{c.st};
  return step_qkv(c, x, qkv, w);
}

ptl_status ptl_attention(const void* qkv, void* attn, const int32_t* cu_seqlens, int32_t num_users,
                         int64_t total_tokens, ptl_dtype dt, void* workspace, size_t ws_bytes,
                         void* stream) {
  ApiRange nvtx_range{"ptl_attention"};
  Call c;
  ptl_status s = setup(&c, total_tokens, num_users, dt, workspace, ws_bytes, stream);
  if (s != PTL_OK) return s;
  if (total_tokens == 0) return PTL_OK;
  if (!qkv || !attn || !cu_seqlens) return PTL_ERR_NULL;
  if (!a16(qkv) || !a16(attn) || !a4(cu_seqlens)) return PTL_ERR_ALIGN;
  if ((s = device_ok()) != PTL_OK) return s;
  if ((s = begin(c)) != PTL_OK) return s;
  EndMark end_mark{c.st};
  mark(c.st, PTL_KERNEL_WORKLIST);
  PTL_TRY(launch_worklist(cu_seqlens, num_users, c.T, c.L, c.ws, c.st));
  return step_attention(c, qkv, attn, cu_seqlens);
}

ptl_status ptl_attention_masked(const void* qkv, void* attn, const int32_t* cu_seqlens,
                                int32_t num_users, int64_t total_tokens, ptl_dtype dt,
                                const ptl_attn_mask* mask, void* workspace, size_t ws_bytes,
                                void* stream) {
  ApiRange nvtx_range{"ptl_attention_masked"};
  Call c;
  ptl_status s = setup(&c, total_tokens, num_users, dt, workspace, ws_bytes, stream);
  if (s != PTL_OK) return s;
  if (!mask) return PTL_ERR_NULL;
  if (mask->target_group_size < 1 || (mask->causal != 0 && mask->causal != 1)) return PTL_ERR_BAD_MASK;
  if (total_tokens == 0) return PTL_OK;
  if (!qkv || !attn || !cu_seqlens) return PTL_ERR_NULL;
  if (!a16(qkv) || !a16(attn) || !a4(cu_seqlens) || (mask->num_contexts && !a4(mask->num_contexts)) ||
      (mask->num_targets && !a4(mask->num_targets)))
    return PTL_ERR_ALIGN;
  if ((s = device_ok()) != PTL_OK) return s;
  if ((s = begin(c)) != PTL_OK) return s;
  const AttnMask m{mask->num_contexts, mask->num_targets, mask->causal, mask->target_group_size,
                   mask->window};
  EndMark end_mark{c.st};
  mark(c.st, PTL_KERNEL_WORKLIST);
  PTL_TRY(launch_worklist(cu_seqlens, num_users, c.T, c.L, c.ws, c.st, &m));
  return step_attention(c, qkv, attn, cu_seqlens, &m);
}

ptl_status ptl_out_projection(const void* attn, const void* x, void* x1, int64_t total_tokens,
                              ptl_dtype dt, const ptl_layer_weights* w, void* workspace, size_t ws_bytes,
                              void* stream) {
  ApiRange nvtx_range{"ptl_out_projection"};
  Call c;
  ptl_status s = setup(&c, total_tokens, 1, dt, workspace, ws_bytes, stream);
  if (s != PTL_OK) return s;
  if (total_tokens == 0) return PTL_OK;
  if (!attn || !x || !x1 || !w || !w->w_o) return PTL_ERR_NULL;
  if (!a16(attn) || !a16(x) || !a16(x1) || !a16(w->w_o) || !opt16(w->b_o)) return PTL_ERR_ALIGN;
  if ((s = device_ok()) != PTL_OK) return s;
  if ((s = begin(c)) != PTL_OK) return s;
  EndMark end_mark{c.st};
  return step_out(c, attn, x, x1, w);
}

ptl_status ptl_gate(const void* x1, void* xn2, int32_t* topk_idx, float* topk_w, int64_t total_tokens,
                    ptl_dtype dt, const ptl_layer_weights* w, void* workspace, size_t ws_bytes,
                    void* stream) {
  ApiRange nvtx_range{"ptl_gate"};
  Call c;
  ptl_status s = setup(&c, total_tokens, 1, dt, workspace, ws_bytes, stream);
  if (s != PTL_OK) return s;
  if (total_tokens == 0) return PTL_OK;
  if (!x1 || !xn2 || !topk_idx || !topk_w || !w || !w->ln2_g || !w->ln2_b || !w->w_gate)
    return PTL_ERR_NULL;
  if (!a16(x1) || !a16(xn2) || !a8(topk_idx) || !a8(topk_w) || !a16(w->ln2_g) || !a16(w->ln2_b) ||
      !a16(w->w_gate) || !opt16(w->b_gate))
    return PTL_ERR_ALIGN;
  if ((s = device_ok()) != PTL_OK) return s;
  if ((s = begin(c)) != PTL_OK) return s;
  EndMark end_mark{c.st};
  return step_gate(c, x1, xn2, topk_idx, topk_w, w);
}

ptl_status ptl_route_build(const int32_t* topk_idx, int64_t total_tokens, int32_t* perm,
                           int32_t* expert_off, void* workspace, size_t ws_bytes, void* stream) {
  ApiRange nvtx_range{"ptl_route_build"};
  Call c;
  ptl_status s = setup(&c, total_tokens, 1, PTL_BF16, workspace, ws_bytes, stream);
  if (s != PTL_OK) return s;
  if (total_tokens == 0) return PTL_OK;
  if (!topk_idx) return PTL_ERR_NULL;
  if (!a4(topk_idx) || (perm && !a4(perm)) || (expert_off && !a4(expert_off))) return PTL_ERR_ALIGN;
  if ((s = device_ok()) != PTL_OK) return s;
  if ((s = begin(c)) != PTL_OK) return s;
  EndMark end_mark{c.st};
  mark(c.st, PTL_KERNEL_ROUTE);
  PTL_TRY(launch_chunk_hist(topk_idx, c.T, at<int32_t>(c, c.L.chunk_cnt), c.err, c.st));
  PTL_TRY(launch_route(topk_idx, c.T, c.L, c.ws, perm, expert_off, nullptr, c.st));
  return PTL_OK;
}

ptl_status ptl_moe(const void* xn2, const int32_t* topk_idx, const float* topk_w, const void* residual,
                   void* out, int64_t total_tokens, ptl_dtype dt, const ptl_layer_weights* w,
                   void* workspace, size_t ws_bytes, void* stream) {
  ApiRange nvtx_range{"ptl_moe"};
  Call c;
  ptl_status s = setup(&c, total_tokens, 1, dt, workspace, ws_bytes, stream);
  if (s != PTL_OK) return s;
  if (total_tokens == 0) return PTL_OK;
  if (!xn2 || !topk_idx || !topk_w || !residual || !out || !w || !w->w1 || !w->w2) return PTL_ERR_NULL;
  if (!a16(xn2) || !a4(topk_idx) || !a4(topk_w) || !a16(residual) || !a16(out) || !a16(w->w1) ||
      !a16(w->w2) || !opt16(w->b1) || !opt16(w->b2))
    return PTL_ERR_ALIGN;
  if ((s = device_ok()) != PTL_OK) return s;
  if ((s = begin(c)) != PTL_OK) return s;
  EndMark end_mark{c.st};
  mark(c.st, PTL_KERNEL_ROUTE);
  PTL_TRY(launch_chunk_hist(topk_idx, c.T, at<int32_t>(c, c.L.chunk_cnt), c.err, c.st));
  return step_moe(c, xn2, topk_idx, topk_w, residual, out, w, nullptr, nullptr);
}

ptl_status ptl_head(const void* h, const ptl_head_weights* head, const uint8_t* pred_mask, float* probs,
                    int32_t* n_pred, int64_t total_tokens, ptl_dtype dt, void* workspace,
                    size_t ws_bytes, void* stream) {
  ApiRange nvtx_range{"ptl_head"};
  Call c;
  ptl_status s = setup(&c, total_tokens, 1, dt, workspace, ws_bytes, stream);
  if (s != PTL_OK) return s;
  if (total_tokens == 0) return PTL_OK;
  if (!h || !head || !pred_mask || !probs) return PTL_ERR_NULL;
  if ((s = check_head(head)) != PTL_OK) return s;
  if (!a16(h) || !a4(probs) || (n_pred && !a4(n_pred))) return PTL_ERR_ALIGN;
  if ((s = device_ok()) != PTL_OK) return s;
  if ((s = begin(c)) != PTL_OK) return s;
  EndMark end_mark{c.st};
  mark(c.st, PTL_KERNEL_HEAD);
  PTL_TRY(launch_head(h, head, pred_mask, probs, n_pred, c.T, c.dt, c.L, c.ws, c.st));
  return PTL_OK;
}

size_t ptl_rep_encoder_workspace_size(int64_t max_tokens, ptl_dtype dt) {
  if (max_tokens < 0 || max_tokens >= (int64_t(1) << 31) || (dt != PTL_F32 && dt != PTL_BF16)) return 0;
  const size_t es = dt == PTL_BF16 ? 2 : 4;
  return 256 + align_up(size_t(max_tokens) * REP_W * es, 256);
}

ptl_status ptl_rep_encoder(const int64_t* ids, int64_t num_ids, const int64_t* bag_offsets,
                           int64_t total_tokens, ptl_dtype dt, const ptl_rep_encoder_weights* w,
                           void* out, void* workspace, size_t ws_bytes, void* stream) {
  ApiRange nvtx_range{"ptl_rep_encoder"};
  if (dt != PTL_F32 && dt != PTL_BF16) return PTL_ERR_DTYPE;
  if (total_tokens < 0 || total_tokens >= (int64_t(1) << 31) || num_ids < 0) return PTL_ERR_SHAPE;
  if (!w || !workspace || !bag_offsets || !out) return PTL_ERR_NULL;
  if (num_ids > 0 && !ids) return PTL_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PTL_ERR_ALIGN;
  if (ws_bytes < ptl_rep_encoder_workspace_size(total_tokens, dt)) return PTL_ERR_WORKSPACE;
  if (!w->ln_g || !w->ln_b || !w->w) return PTL_ERR_NULL;
  if (!a16(out) || !a16(w->w) || !a16(w->ln_g) || !a16(w->ln_b) || !a4(bag_offsets) || (ids && !a4(ids)))
    return PTL_ERR_ALIGN;
  RepTables tb;
  for (int s = 0; s < REP_SLOTS; ++s) {
    if (w->vocab[s] < 0) return PTL_ERR_SHAPE;
    if (w->vocab[s] > 0 && !w->tables[s]) return PTL_ERR_NULL;
    if (!a16(w->tables[s])) return PTL_ERR_ALIGN;
    tb.t[s] = w->tables[s];
    tb.vocab[s] = w->vocab[s];
  }
  if (total_tokens == 0) return PTL_OK;
  ptl_status s;
  if ((s = device_ok()) != PTL_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  int32_t* err = reinterpret_cast<int32_t*>(ws);
  char* normed = ws + 256;
  const int T = int(total_tokens);
  if (cudaMemsetAsync(err, 0, sizeof(int32_t), st) != cudaSuccess) return PTL_ERR_CUDA;
  mark(st, PTL_KERNEL_LAYERNORM);
  PTL_TRY(launch_embag_ln(tb, ids, bag_offsets, num_ids, T, w->ln_g, w->ln_b, normed, dt, err, st));
  EndMark end_mark{st};
  if (dt == PTL_BF16) {
    CUtensorMap ma, mb, mo;
    if (!map_bf16(&ma, normed, REP_W, uint64_t(T), REP_W * 2, 64, 128)) return PTL_ERR_CUDA;
    if (!map_bf16(&mb, w->w, REP_W, D, REP_W * 2, 64, 128)) return PTL_ERR_CUDA;
    if (!map_bf16(&mo, out, D, uint64_t(T), D * 2, 64, 128)) return PTL_ERR_CUDA;
    mark(st, PTL_KERNEL_GEMM_QKV);
    PTL_TRY(launch_gemm_rep(ma, mb, mo, w->b, T, err, st));
  } else {
    WsLayout L{};  // the fp32 GEMM reads only the error word (offset 0) in this mode
    mark(st, PTL_KERNEL_GEMM_QKV);
    PTL_TRY(launch_gemm_f32(0, reinterpret_cast<const float*>(normed), REP_W, F32(w->w), w->b, nullptr,
                            static_cast<float*>(out), D, T, D, REP_W, L, ws, st));
  }
  return PTL_OK;
}

ptl_status ptl_quantize_rows_e4m3(const void* x, ptl_dtype dt, int64_t rows, int32_t cols, uint8_t* codes,
                                  float* scales, void* stream) {
  ApiRange nvtx_range{"ptl_quantize_rows_e4m3"};
  if (dt != PTL_F32 && dt != PTL_BF16) return PTL_ERR_DTYPE;
  if (rows < 0 || cols < 16 || cols % 16 != 0) return PTL_ERR_SHAPE;
  if (rows == 0) return PTL_OK;
  if (!x || !codes || !scales) return PTL_ERR_NULL;
  if (!a16(x) || !a16(codes) || !a4(scales)) return PTL_ERR_ALIGN;
  ptl_status s;
  if ((s = device_ok()) != PTL_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  EndMark end_mark{st};
  mark(st, PTL_KERNEL_LAYERNORM);
  PTL_TRY(launch_quant_rows_e4m3(x, dt, rows, cols, codes, scales, st));
  return PTL_OK;
}

ptl_status ptl_linear_fp8(const uint8_t* xq, const float* sx, const uint8_t* wq, const float* sw,
                          const float* bias, void* out, int64_t rows, int32_t in_features,
                          int32_t out_features, void* workspace, size_t ws_bytes, void* stream) {
  ApiRange nvtx_range{"ptl_linear_fp8"};
  if (rows < 0 || rows >= (int64_t(1) << 31) || in_features < 128 || in_features % 128 != 0 ||
      out_features < 256 || out_features % 256 != 0)
    return PTL_ERR_SHAPE;
  if (!workspace) return PTL_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PTL_ERR_ALIGN;
  if (ws_bytes < 256) return PTL_ERR_WORKSPACE;
  if (rows == 0) return PTL_OK;
  if (!xq || !sx || !wq || !sw || !out) return PTL_ERR_NULL;
  if (!a16(xq) || !a16(wq) || !a16(out) || !a4(sx) || !a4(sw) || !opt16(bias)) return PTL_ERR_ALIGN;
  ptl_status s;
  if ((s = device_ok()) != PTL_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* err = static_cast<int32_t*>(workspace);
  CUtensorMap ma, mb, mo;
  if (!map_u8(&ma, xq, uint64_t(in_features), uint64_t(rows), uint64_t(in_features), 128)) return PTL_ERR_CUDA;
  if (!map_u8(&mb, wq, uint64_t(in_features), uint64_t(out_features), uint64_t(in_features), 128))
    return PTL_ERR_CUDA;
  if (!map_bf16(&mo, out, uint64_t(out_features), uint64_t(rows), uint64_t(out_features) * 2, 64, 128))
    return PTL_ERR_CUDA;
  mark(st, PTL_KERNEL_CLEAR);
  if (cudaMemsetAsync(err, 0, sizeof(int32_t), st) != cudaSuccess) return PTL_ERR_CUDA;
  EndMark end_mark{st};
  mark(st, PTL_KERNEL_GEMM_QKV);
  PTL_TRY(launch_gemm_fp8(ma, mb, mo, sx, sw, bias, int(rows), out_features, in_features, err, st));
  return PTL_OK;
}

ptl_status ptl_wait_selftest(void* workspace, size_t ws_bytes, int32_t which, int64_t limit_ns,
                             void* stream) {
  ApiRange nvtx_range{"ptl_wait_selftest"};
  if (!workspace) return PTL_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PTL_ERR_ALIGN;
  if (ws_bytes < 256) return PTL_ERR_WORKSPACE;
  if ((which != 0 && which != 1) || limit_ns < 1000 || limit_ns > 1000000000) return PTL_ERR_SHAPE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  // the flag lives in the error block's spare bytes; nothing else writes it
  int32_t* flag = reinterpret_cast<int32_t*>(ws + 128);
  if (cudaMemsetAsync(flag, 0, sizeof(int32_t), st) != cudaSuccess) return PTL_ERR_CUDA;
  if (launch_wait_selftest(reinterpret_cast<int32_t*>(ws), flag, which, uint64_t(limit_ns), st) != 0)
    return PTL_ERR_CUDA;
  return PTL_OK;
}

ptl_status ptl_last_device_error(void* workspace, size_t ws_bytes, void* stream) {
  if (!workspace) return PTL_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PTL_ERR_ALIGN;
  if (ws_bytes < 256) return PTL_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return PTL_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return PTL_ERR_CUDA;
  if (cudaMemset(workspace, 0, sizeof(v)) != cudaSuccess) return PTL_ERR_CUDA;
  return static_cast<ptl_status>(v);
}

}  // extern "C"
