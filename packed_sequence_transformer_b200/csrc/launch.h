// launch.h -- host-side launchers of the layer's kernels (internal to libptl).
// Each returns 0 on success and -1 when the launch (or its configuration)
// failed.  All launches are asynchronous on `st`.
#pragma once
#include <cstdint>
#include <mutex>
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace ptl {

// A value set up once per device (kernel attributes such as the dynamic
// shared-memory limit, and launch-shape queries, belong to a device, not to
// the process).  get() returns the current device's value, running init()
// on the first call for that device (under a lock); a failed init (<= 0) is
// not remembered, so the next call tries again.  Returns -1 on failure.
constexpr int kMaxDevices = 64;
struct PerDevice {
  std::mutex mu;
  int v[kMaxDevices] = {};
  template <typename F>
  int get(F&& init) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
    std::lock_guard<std::mutex> lock(mu);
    if (v[dev] <= 0) {
      const int r = init();
      if (r <= 0) return -1;
      v[dev] = r;
    }
    return v[dev];
  }
};

// Tracing hooks (api.cu): trace_mark opens the NVTX range of a kernel launch
// of `kind` and records the calling thread's trace event for it (no-ops
// without a profiler or an installed trace); ApiRange is the NVTX range of an
// entry point, closing both on every return path; EndMark records the
// closing PTL_KERNEL_END event when the entry point returns.
void trace_mark(cudaStream_t st, int kind);
void api_range_push(const char* name);
void api_range_pop();
struct ApiRange {
  explicit ApiRange(const char* name) { api_range_push(name); }
  ~ApiRange() { api_range_pop(); }
  ApiRange(const ApiRange&) = delete;
  ApiRange& operator=(const ApiRange&) = delete;
};
struct EndMark {
  cudaStream_t st;
  ~EndMark() { trace_mark(st, PTL_KERNEL_END); }
};

// Launches `kernel` on `st` with programmatic stream serialization, so a
// captured graph gets programmatic edges and the kernel may launch while its
// predecessor drains (the kernels call pdl_trigger / pdl_wait).
template <typename... KArgs, typename... Args>
inline int launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                    Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) == cudaSuccess ? 0 : -1;
}

constexpr int QKV_BN = 192;
constexpr int OUT_BN = 256;
constexpr int MOE1_BN = 256;

// kernels_simt.cu
int num_sms();  // of the current device (148 when it cannot be queried)
// A kernel whose bounded wait runs out (which: 0 mbarrier, 1 global flag).
int launch_wait_selftest(int32_t* err, const int32_t* flag, int which, uint64_t limit_ns,
                         cudaStream_t st);
// mask (nullable): HSTU-style variant; validates the per-user counts and
// lists the units for the masked attention
int launch_worklist(const int32_t* cu, int U, int T, const WsLayout& L, char* ws, cudaStream_t st,
                    const AttnMask* mask = nullptr);
int launch_layernorm(const void* x, const float* g, const float* b, void* y, int T, ptl_dtype dt,
                     cudaStream_t st);
// bf16 layer / stack: the work list (block 0), with a prediction mask each
// kept token's slot in the head's compacted output and their count (block
// 1, into the workspace's head_p and *n_pred), and the first layer's
// LayerNorm1 of x into y (the other blocks) in one launch
int launch_prologue(const int32_t* cu, int U, int T, const WsLayout& L, char* ws, const void* x, const float* g,
                    const float* b, void* y, cudaStream_t st, const uint8_t* pred_mask = nullptr,
                    int32_t* n_pred = nullptr);
int launch_gate(const void* x1, const float* g, const float* b, const float* wg, const float* bg,
                void* xn2, int32_t* idx, float* w, int32_t* chunk_cnt, int T, ptl_dtype dt,
                cudaStream_t st);
int launch_chunk_hist(const int32_t* idx, int T, int32_t* chunk_cnt, int32_t* err, cudaStream_t st);
// bf16 layer path: gate + route builder in one kernel (idx, wgt, pos, xperm,
// tiles, meta in the workspace; the look-back state must be zero)
int launch_gate_route(const void* x1, const float* g, const float* b, const float* wg, const float* bg,
                      int T, const WsLayout& L, char* ws, cudaStream_t st);
// perm / expert_off (either may be NULL) of the fused path
int launch_route_debug(int T, const WsLayout& L, const char* ws, int32_t* perm, int32_t* expert_off,
                       cudaStream_t st);
// xn2 (bf16 build, nullable): also copy each route's LayerNorm2 row to its
// padded slot of the workspace's xperm
int launch_route(const int32_t* idx, int T, const WsLayout& L, char* ws, int32_t* dbg_perm,
                 int32_t* dbg_off, const void* xn2, cudaStream_t st);
// The prediction head as its own launches (the fp32 stack and ptl_head):
// every token's probability into head_p, then the kept ones compacted
int launch_head(const void* h, const ptl_head_weights* hw, const uint8_t* mask, float* probs,
                int32_t* n_pred, int T, ptl_dtype dt, const WsLayout& L, char* ws, cudaStream_t st);
int launch_gemm_f32(int mode, const float* A, int lda, const float* W, const float* bias,
                    const float* R, float* C, int ldc, int M, int N, int Kd, const WsLayout& L,
                    const char* ws, cudaStream_t st);
// ln_g / ln_b / xn: optional (all NULL or none) LayerNorm of the output row into xn.
// streamed_after (nullable): the fused expert GEMMs of that workspace layout run
// just before; the combine starts on their finished tiles instead of waiting
// for the whole launch
// The prediction head computed by the last layer's combine (bf16 stack):
// LayerNorm_f parameters g, b, the weight row w, bias (nullable), the output
// probs and each token's slot in it (-1: not predicted).
struct HeadArgs {
  const float *g, *b, *w, *bias;
  float* probs;
  const int32_t* slot;
};
int launch_combine_bf16(const void* ybuf, const int32_t* pos, const float* w, const float* x1, void* out,
                        int T, const float* ln_g, const float* ln_b, void* xn, int32_t* err,
                        cudaStream_t st, const WsLayout* streamed_after = nullptr, const char* ws = nullptr,
                        const HeadArgs* head = nullptr);
int launch_combine_f32(const float* y, const float* w, const float* x1, float* out, int T,
                       const int32_t* err, cudaStream_t st);
int launch_attn_f32(const float* qkv, float* out, const int32_t* cu, const WsLayout& L,
                    const char* ws, cudaStream_t st, const AttnMask* mask = nullptr);

// Per-row e4m3 codes [rows][cols] and float32 scales [rows] of x (dt)
int launch_quant_rows_e4m3(const void* x, ptl_dtype dt, int64_t rows, int cols, uint8_t* codes, float* scales,
                           cudaStream_t st);

// RepEncoder: embedding bags + LayerNorm(14336) into out [T][14336] (dt)
int launch_embag_ln(const RepTables& tb, const int64_t* ids, const int64_t* off, int64_t n_ids, int T,
                    const float* g, const float* b, void* out, ptl_dtype dt, int32_t* err,
                    cudaStream_t st);

// gemm_tc.cu (bf16, tcgen05).  QKV and the output projection run on CTA
// pairs: their B (weight) tensor maps have boxes of BN/2 rows.
// pf0 / pf1 (nullable): weights of later kernels of the layer that the QKV
// GEMM's CTAs bring into L2 before their inputs are ready
int launch_gemm_qkv(const CUtensorMap& xn, const CUtensorMap& w, const CUtensorMap& qkv_out,
                    const float* bias, void* qkv, int T, int32_t* err, cudaStream_t st,
                    const void* pf0 = nullptr, size_t pf0_bytes = 0, const void* pf1 = nullptr,
                    size_t pf1_bytes = 0);
int launch_gemm_out(const CUtensorMap& attn, const CUtensorMap& w, const CUtensorMap& x1_out,
                    const float* bias, const void* x, void* x1, int T, int32_t* err, cudaStream_t st);
// RepEncoder Linear: out [T][512] = normed [T][14336] W^T + b (256 x 256 pair tiles)
int launch_gemm_rep(const CUtensorMap& normed, const CUtensorMap& w, const CUtensorMap& out_map,
                    const float* bias, int T, int32_t* err, cudaStream_t st);
int launch_gemm_moe1(const CUtensorMap& xperm, const CUtensorMap& w1, const CUtensorMap& hbuf_out,
                     const float* b1, const WsLayout& L, char* ws, cudaStream_t st);
// Both expert GEMMs in one persistent launch (first-GEMM tiles, then
// second-GEMM tiles, each waiting for its M tile's hidden rows); the
// workspace's per-M-tile counters (moe_done) must be zero.
int launch_gemm_moe12(const CUtensorMap& xperm, const CUtensorMap& w1, const CUtensorMap& hbuf,
                      const CUtensorMap& w2, const CUtensorMap& ybuf_out, const float* b1, const float* b2,
                      const WsLayout& L, char* ws, cudaStream_t st);
int launch_gemm_moe2(const CUtensorMap& hbuf, const CUtensorMap& w2, const CUtensorMap& ybuf_out,
                     const float* b2, const WsLayout& L, char* ws, cudaStream_t st);

// FP8: out [M][N] bf16 = (xq [M][K] wq [N][K]^T) * sx[m] * sw[n] + b[n], e4m3
// codes with per-row scales, 256 x 256 pair tiles (K a multiple of 128, N of 256)
int launch_gemm_fp8(const CUtensorMap& xq, const CUtensorMap& wq, const CUtensorMap& out_map, const float* sx,
                    const float* sw, const float* bias, int M, int N, int Kd, int32_t* err, cudaStream_t st);

// attn_tc.cu (bf16, tcgen05)
// mask (nullable): the HSTU-style variant, over a work list built with the
// same mask
// list_early: the work list was written by a kernel that completed before
// the attention's own predecessor passed its dependency wait (the layer
// path), so the kernel reads its list heads before its own wait.
int launch_attn_tc(const CUtensorMap& qkv_map, void* out, const int32_t* cu, const WsLayout& L,
                   char* ws, cudaStream_t st, const AttnMask* mask = nullptr, bool list_early = false);

}  // namespace ptl
