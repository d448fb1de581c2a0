// noalloc.cu -- jagged causal attention for callers that cannot allocate
// device memory.
//
// Some host programs own every byte of device memory through their own pool
// or budget and give a library no allocator, and some latency-critical
// loops cannot afford cudaMalloc, which may synchronise the device.  This
// entry point serves them: it computes what ptl_attention computes, but the
// only scratch it needs -- the device error word and the (user, query block)
// work list -- lives in one fixed array in the library's own device memory
// instead of a caller-provided workspace.  Each GPU that loads the library
// holds the array until the process exits.
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/ptl.h"
#include "common.cuh"
#include "launch.h"

namespace {
using namespace ptl;

// Scratch for the attention work list and the error word (the leading part
// of the workspace layout, up to the first activation buffer).  Sized for
// PTL_NOALLOC_MAX_TOKENS tokens and PTL_NOALLOC_MAX_USERS users.
static __device__ __align__(256) unsigned char g_noalloc_scratch[PTL_NOALLOC_SCRATCH_BYTES];

std::mutex g_addr_mu;
void* g_addr[kMaxDevices];

// Host code cannot pass `g_noalloc_scratch` itself to a kernel: in host code
// that name is a host-side stand-in, not a device address.  The address is
// looked up once per device, with that device current, and cached.
ptl_status scratch_on_current_device(char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PTL_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PTL_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_addr_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return PTL_ERR_CUDA;
    g_addr[dev] = p;
  }
  *out = static_cast<char*>(g_addr[dev]);
  return PTL_OK;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// TMA descriptor of the packed qkv rows: 1536 bf16 columns, 128 x 64 boxes.
bool qkv_map(CUtensorMap* m, const void* qkv, int T) {
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
  if (!fn) return false;
  const cuuint64_t dims[2] = {cuuint64_t(QKV_N), cuuint64_t(T)};
  const cuuint64_t strides[1] = {cuuint64_t(QKV_N) * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(qkv), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" ptl_status ptl_attention_noalloc(const void* qkv, void* attn, const int32_t* cu_seqlens,
                                            int32_t num_users, int64_t total_tokens, ptl_dtype dt,
                                            int32_t* device_status, void* stream) {
  ApiRange nvtx_range{"ptl_attention_noalloc"};
  if (dt != PTL_F32 && dt != PTL_BF16) return PTL_ERR_DTYPE;
  if (num_users < 1 || total_tokens < 0) return PTL_ERR_SHAPE;
  if (total_tokens > PTL_NOALLOC_MAX_TOKENS || num_users > PTL_NOALLOC_MAX_USERS) return PTL_ERR_SHAPE;
  if (total_tokens == 0) return PTL_OK;
  if (!qkv || !attn || !cu_seqlens) return PTL_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(qkv) & 15u) || (reinterpret_cast<uintptr_t>(attn) & 15u) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) ||
      (reinterpret_cast<uintptr_t>(device_status) & 3u))
    return PTL_ERR_ALIGN;
  WsLayout L;
  if (!make_layout(total_tokens, num_users, dt, &L)) return PTL_ERR_SHAPE;
  if (L.wl_end > sizeof(g_noalloc_scratch)) return PTL_ERR_SHAPE;  // work list must fit the array
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return PTL_ERR_CUDA;
  if (major != 10) return PTL_ERR_UNSUPPORTED;
  char* ws = nullptr;
  ptl_status s = scratch_on_current_device(&ws);
  if (s != PTL_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int T = int(total_tokens);
  // The array keeps the previous call's contents: the error word must start
  // at zero (the work-list kernel clears its own counters).
  trace_mark(st, PTL_KERNEL_CLEAR);
  if (cudaMemsetAsync(ws + L.err, 0, sizeof(int32_t), st) != cudaSuccess) return PTL_ERR_CUDA;
  EndMark end_mark{st};
  trace_mark(st, PTL_KERNEL_WORKLIST);
  if (launch_worklist(cu_seqlens, num_users, T, L, ws, st) != 0) return PTL_ERR_CUDA;
  CUtensorMap m;
  if (dt == PTL_BF16 && !qkv_map(&m, qkv, T)) return PTL_ERR_CUDA;
  trace_mark(st, PTL_KERNEL_ATTENTION);
  if (dt == PTL_BF16) {
    if (launch_attn_tc(m, attn, cu_seqlens, L, ws, st) != 0) return PTL_ERR_CUDA;
  } else {
    if (launch_attn_f32(static_cast<const float*>(qkv), static_cast<float*>(attn), cu_seqlens, L, ws,
                        st) != 0)
      return PTL_ERR_CUDA;
  }
  if (device_status) trace_mark(st, PTL_KERNEL_COPY);
  if (device_status &&
      cudaMemcpyAsync(device_status, ws + L.err, sizeof(int32_t), cudaMemcpyDeviceToDevice, st) !=
          cudaSuccess)
    return PTL_ERR_CUDA;
  return PTL_OK;
}
