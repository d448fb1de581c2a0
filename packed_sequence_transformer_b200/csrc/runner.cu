// runner.cu -- the layer stack as one CUDA graph per token bucket.
//
// Issued kernel by kernel, the serving loop is launch-bound (Days-gone/cti2026
// README, CUDA Graph section: a few hundred launches per batch, most of the
// host time spent issuing them).  The cure there is CUDA graph replay with
// bucketed static shapes: every batch is padded up to a bucket of the token
// count, the stack is captured once per bucket over static buffers, and a
// batch becomes a handful of copies plus one graph launch, with no host
// synchronisation.  This file is that runtime, on top of ptl_stack_forward
// (whose kernels chain with programmatic dependent launch inside the graph).
//
// Padding.  A batch of T tokens / U users runs in the bucket of Tb tokens
// (T rounded up to the bucket stride) and a fixed Ub = max_users +
// ceil((stride - 1) / 128) users: the U real users first, then padding users
// of at most 128 zero tokens each covering T .. Tb (one query block each, so
// the padding costs the least attention work), then zero-length users up to
// Ub.  Users are independent and every other step is per token, so the real
// rows come out exactly as from a direct ptl_stack_forward call on the
// unpadded batch; padding tokens have pred_mask 0 and never reach probs.
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/ptl.h"
#include "common.cuh"

namespace ptl {

// Pads a batch of T tokens / U users to the bucket of Tb tokens / Ub users
// in the static buffers: zero-fills the padding rows of x (row_bytes each)
// and of the prediction mask (nullable), and (block 0) writes the padding
// users' offsets cu[U + 1 .. Ub].  The real offsets cu[0 .. U] were copied in
// before; if cu[U] is not T the batch is malformed, and the kernel makes the
// offsets end below Tb so that the stack's offset validator reports
// PTL_ERR_BAD_OFFSETS (the error word itself is cleared by the stack call,
// so the fault has to travel through the offsets).
__global__ void pad_batch_kernel(int32_t* cu, int U, int T, int Tb, int Ub, char* x,
                                 int row_bytes, uint8_t* mask) {
  pdl_wait();
  pdl_trigger();
  const size_t n16 = size_t(Tb - T) * size_t(row_bytes) / 16;
  int4* xp = reinterpret_cast<int4*>(x + size_t(T) * size_t(row_bytes));
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += size_t(gridDim.x) * blockDim.x)
    xp[i] = make_int4(0, 0, 0, 0);
  if (mask)
    for (int i = T + int(blockIdx.x * blockDim.x + threadIdx.x); i < Tb; i += gridDim.x * blockDim.x)
      mask[i] = 0;
  if (blockIdx.x != 0) return;
  const bool bad = cu[U] != T;
  for (int i = U + 1 + int(threadIdx.x); i <= Ub; i += blockDim.x) {
    const int64_t v = int64_t(T) + int64_t(i - U) * ATT_BLK;
    cu[i] = v < Tb ? int32_t(v) : Tb;
  }
  __syncthreads();
  if (bad && threadIdx.x == 0) cu[Ub] = -1;
}

}  // namespace ptl

struct ptl_stack_runner {
  int device = 0;
  int64_t max_tokens = 0, tmax = 0;
  int32_t max_users = 0, ub = 0, stride = 0, n_layers = 0;
  ptl_dtype dt = PTL_BF16;
  size_t es = 2;
  std::vector<ptl_layer_weights> layers;
  bool has_head = false;
  ptl_head_weights head{};
  char* mem = nullptr;  // one allocation, carved below
  char* ws = nullptr;
  size_t ws_bytes = 0;
  char* x_s = nullptr;
  char* out_s = nullptr;
  int32_t* cu_s = nullptr;
  uint8_t* mask_s = nullptr;
  float* probs_s = nullptr;
  int32_t* npred_s = nullptr;
  cudaStream_t cap = nullptr;  // capture only; nothing executes on it
  std::vector<cudaGraphExec_t> exec;
  std::mutex mu;
};

namespace {

int32_t pad_users(int32_t stride) { return (stride - 1 + ptl::ATT_BLK - 1) / ptl::ATT_BLK; }

int64_t bucket_tokens(int64_t T, int32_t stride) { return (T + stride - 1) / stride * stride; }

bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool a4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

void release(ptl_stack_runner* r) {
  for (cudaGraphExec_t e : r->exec)
    if (e) cudaGraphExecDestroy(e);
  if (r->mem) cudaFree(r->mem);
  if (r->cap) cudaStreamDestroy(r->cap);
  delete r;
}

// Captures the stack for bucket b (Tb tokens, Ub users) over the static
// buffers and instantiates it.
ptl_status capture(ptl_stack_runner* r, int b, cudaGraphExec_t* out) {
  const int64_t Tb = int64_t(b + 1) * r->stride;
  if (cudaStreamBeginCapture(r->cap, cudaStreamCaptureModeThreadLocal) != cudaSuccess)
    return PTL_ERR_CUDA;
  const ptl_status s = ptl_stack_forward(
      r->x_s, r->out_s, r->cu_s, r->ub, Tb, r->n_layers, r->dt, r->layers.data(),
      r->has_head ? &r->head : nullptr, r->has_head ? r->mask_s : nullptr,
      r->has_head ? r->probs_s : nullptr, r->has_head ? r->npred_s : nullptr, r->ws, r->ws_bytes,
      r->cap);
  cudaGraph_t g = nullptr;
  const cudaError_t e = cudaStreamEndCapture(r->cap, &g);
  if (s != PTL_OK || e != cudaSuccess) {
    if (g) cudaGraphDestroy(g);
    return s != PTL_OK ? s : PTL_ERR_CUDA;
  }
  const cudaError_t ie = cudaGraphInstantiate(out, g, 0);
  cudaGraphDestroy(g);
  return ie == cudaSuccess ? PTL_OK : PTL_ERR_CUDA;
}

ptl_status graph_for(ptl_stack_runner* r, int b, cudaGraphExec_t* out) {
  std::lock_guard<std::mutex> lock(r->mu);
  if (!r->exec[b]) {
    const ptl_status s = capture(r, b, &r->exec[b]);
    if (s != PTL_OK) {
      r->exec[b] = nullptr;
      return s;
    }
  }
  *out = r->exec[b];
  return PTL_OK;
}

}  // namespace

extern "C" {

ptl_status ptl_runner_bucket(int64_t total_tokens, int32_t max_users, int32_t stride,
                             int64_t* bucket, int32_t* padded_users) {
  if (!bucket || !padded_users) return PTL_ERR_NULL;
  if (stride == 0) stride = PTL_RUNNER_STRIDE;
  if (stride < 0 || stride % ptl::ATT_BLK != 0 || total_tokens < 0 || max_users < 1 ||
      total_tokens >= (int64_t(1) << 31) - stride || max_users > (int32_t(1) << 30))
    return PTL_ERR_SHAPE;
  *bucket = bucket_tokens(total_tokens, stride);
  *padded_users = max_users + pad_users(stride);
  return PTL_OK;
}

ptl_status ptl_runner_create(int64_t max_tokens, int32_t max_users, int32_t num_layers, ptl_dtype dt,
                             const ptl_layer_weights* layers, const ptl_head_weights* head,
                             int32_t stride, ptl_stack_runner** runner) {
  if (!runner) return PTL_ERR_NULL;
  *runner = nullptr;
  if (!layers) return PTL_ERR_NULL;
  if (dt != PTL_F32 && dt != PTL_BF16) return PTL_ERR_DTYPE;
  if (num_layers < 1 || max_tokens < 1) return PTL_ERR_SHAPE;
  int64_t tmax = 0;
  int32_t ub = 0;
  ptl_status s = ptl_runner_bucket(max_tokens, max_users, stride, &tmax, &ub);
  if (s != PTL_OK) return s;
  if (stride == 0) stride = PTL_RUNNER_STRIDE;
  ptl_stack_runner* r = new (std::nothrow) ptl_stack_runner();
  if (!r) return PTL_ERR_CUDA;
  r->max_tokens = max_tokens;
  r->tmax = tmax;
  r->max_users = max_users;
  r->ub = ub;
  r->stride = stride;
  r->n_layers = num_layers;
  r->dt = dt;
  r->es = dt == PTL_BF16 ? 2 : 4;
  r->layers.assign(layers, layers + num_layers);
  if (head) {
    r->has_head = true;
    r->head = *head;
  }
  r->exec.assign(size_t(tmax / stride), nullptr);
  if (cudaGetDevice(&r->device) != cudaSuccess) {
    release(r);
    return PTL_ERR_CUDA;
  }
  // one allocation: workspace, x, out, offsets, mask, probs, count
  r->ws_bytes = ptl_workspace_size(tmax, ub, dt);
  if (r->ws_bytes == 0) {
    release(r);
    return PTL_ERR_SHAPE;
  }
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = ptl::align_up(o + bytes, 256);
    return at;
  };
  const size_t o_ws = take(r->ws_bytes);
  const size_t o_x = take(size_t(tmax) * ptl::D * r->es);
  const size_t o_out = take(size_t(tmax) * ptl::D * r->es);
  const size_t o_cu = take(4 * (size_t(ub) + 1));
  const size_t o_mask = take(size_t(tmax));
  const size_t o_probs = take(4 * size_t(tmax));
  const size_t o_np = take(4);
  if (cudaMalloc(&r->mem, o) != cudaSuccess) {
    r->mem = nullptr;
    release(r);
    return PTL_ERR_CUDA;
  }
  r->ws = r->mem + o_ws;
  r->x_s = r->mem + o_x;
  r->out_s = r->mem + o_out;
  r->cu_s = reinterpret_cast<int32_t*>(r->mem + o_cu);
  r->mask_s = reinterpret_cast<uint8_t*>(r->mem + o_mask);
  r->probs_s = reinterpret_cast<float*>(r->mem + o_probs);
  r->npred_s = reinterpret_cast<int32_t*>(r->mem + o_np);
  if (cudaMemset(r->mem, 0, o) != cudaSuccess ||
      cudaStreamCreateWithFlags(&r->cap, cudaStreamNonBlocking) != cudaSuccess) {
    release(r);
    return PTL_ERR_CUDA;
  }
  *runner = r;
  return PTL_OK;
}

ptl_status ptl_runner_capture(ptl_stack_runner* r, int64_t total_tokens) {
  if (!r) return PTL_ERR_NULL;
  if (total_tokens < 1 || total_tokens > r->max_tokens) return PTL_ERR_SHAPE;
  cudaGraphExec_t e = nullptr;
  return graph_for(r, int(bucket_tokens(total_tokens, r->stride) / r->stride) - 1, &e);
}

ptl_status ptl_runner_forward(ptl_stack_runner* r, const void* x, void* out, const int32_t* cu_seqlens,
                              int32_t num_users, int64_t total_tokens, const uint8_t* pred_mask,
                              float* probs, int32_t* n_pred, void* stream) {
  if (!r) return PTL_ERR_NULL;
  if (total_tokens < 0 || total_tokens > r->max_tokens || num_users < 1 || num_users > r->max_users)
    return PTL_ERR_SHAPE;
  if (!x || !cu_seqlens) return PTL_ERR_NULL;
  if (!out && !r->has_head) return PTL_ERR_NULL;
  if (r->has_head && (!pred_mask || !probs)) return PTL_ERR_NULL;
  if (!a16(x) || (out && !a16(out)) || !a4(cu_seqlens) || (probs && !a4(probs)) ||
      (n_pred && !a4(n_pred)))
    return PTL_ERR_ALIGN;
  if (total_tokens == 0) return PTL_OK;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return PTL_ERR_CUDA;
  if (dev != r->device) return PTL_ERR_SHAPE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t T = total_tokens, Tb = bucket_tokens(T, r->stride);
  const int b = int(Tb / r->stride) - 1;
  cudaGraphExec_t g = nullptr;
  ptl_status s = graph_for(r, b, &g);
  if (s != PTL_OK) return s;
  const size_t row = size_t(ptl::D) * r->es;
  // inputs into the static buffers (host or device sources), then one
  // kernel for the padding rows, mask entries and users
  if (cudaMemcpyAsync(r->x_s, x, size_t(T) * row, cudaMemcpyDefault, st) != cudaSuccess)
    return PTL_ERR_CUDA;
  if (cudaMemcpyAsync(r->cu_s, cu_seqlens, 4 * (size_t(num_users) + 1), cudaMemcpyDefault, st) !=
      cudaSuccess)
    return PTL_ERR_CUDA;
  if (r->has_head &&
      cudaMemcpyAsync(r->mask_s, pred_mask, size_t(T), cudaMemcpyDefault, st) != cudaSuccess)
    return PTL_ERR_CUDA;
  {
    const size_t n16 = size_t(Tb - T) * row / 16;
    size_t blocks = (n16 + 255) / 256;
    if (blocks < 1) blocks = 1;
    if (blocks > 64) blocks = 64;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(blocks));
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    if (cudaLaunchKernelEx(&cfg, ptl::pad_batch_kernel, r->cu_s, int(num_users), int(T), int(Tb),
                           int(r->ub), r->x_s, int(row), r->has_head ? r->mask_s : nullptr) !=
        cudaSuccess)
      return PTL_ERR_CUDA;
  }
  if (cudaGraphLaunch(g, st) != cudaSuccess) return PTL_ERR_CUDA;
  // results out of the static buffers (host or device destinations)
  if (out && cudaMemcpyAsync(out, r->out_s, size_t(T) * row, cudaMemcpyDefault, st) != cudaSuccess)
    return PTL_ERR_CUDA;
  if (r->has_head) {
    if (cudaMemcpyAsync(probs, r->probs_s, 4 * size_t(T), cudaMemcpyDefault, st) != cudaSuccess)
      return PTL_ERR_CUDA;
    if (n_pred && cudaMemcpyAsync(n_pred, r->npred_s, 4, cudaMemcpyDefault, st) != cudaSuccess)
      return PTL_ERR_CUDA;
  }
  return PTL_OK;
}

ptl_status ptl_runner_last_device_error(ptl_stack_runner* r, void* stream) {
  if (!r) return PTL_ERR_NULL;
  return ptl_last_device_error(r->ws, r->ws_bytes, stream);
}

int32_t ptl_runner_graphs(const ptl_stack_runner* r) {
  if (!r) return -1;
  int32_t n = 0;
  for (cudaGraphExec_t e : r->exec) n += e != nullptr;
  return n;
}

void ptl_runner_destroy(ptl_stack_runner* r) {
  if (r) release(r);
}

}  // extern "C"
