// gemm_tc.cu -- tcgen05 GEMMs of the layer (bf16 in, fp32 accumulate in TMEM).
//
// One CTA computes a 128 x BN output tile, D = A B^T with A [M][K] and
// B = W [N][K] (nn.Linear layout), both K-major in shared memory with the
// 128-byte swizzle.  Warp roles (6 warps):
//   warp 0      TMA producer: one elected thread streams 64-wide K slices of
//               A and B through a STAGES-deep ring of shared-memory buffers;
//   warp 1      allocates the TMEM accumulator; one thread issues
//               tcgen05.mma (M=128, N=BN, K=16) and commits each stage back
//               to the producer, then the finished accumulator to the epilogue;
//   warps 2..5  epilogue: each thread owns one accumulator row (TMEM lane),
//               reads it with tcgen05.ld and applies the fused epilogue.  In
//               the expert GEMM1 these warps first gather the A rows
//               (token rows of LayerNorm2 output picked through the route
//               permutation) into the swizzled ring themselves.
// Modes:
//   QKV   qkv = xn Wqkv^T + b_qkv                         (A by TMA)
//   OUT   x1  = x + attn Wo^T + b_o, kept in fp32         (A by TMA)
//   MOE1  H[row] = ReLU(xn2[token(row)] W1[e]^T + b1[e])  (A gathered)
//   MOE2  y = H W2[e]^T + b2[e], then the top-2 combine   (A by TMA)
//         out[t] = (x1[t] + w[t,0] y(t,0)) + w[t,1] y(t,1): both routes of
//         a token stage their fp32 y; the second to arrive (per-token
//         atomic counter, no waiting) combines in the fixed k order.
// Every wait is bounded; a timeout sets PTL_ERR_TIMEOUT and unwinds.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace ptl {
using namespace sm100;

struct GemmTcParams {
  int M;                         // rows of A (dense modes)
  int N_total;                   // output columns (per expert in the MoE modes)
  int num_kb;                    // K / 64
  const float* bias;             // [N] or [E][N]; may be NULL
  const __nv_bfloat16* resid;    // OUT: x (row stride 512)
  const float* resid_f32;        // MOE2: x1 in fp32 (row stride 512)
  __nv_bfloat16* out;            // output rows
  float* out_f32;                // OUT: x1 in fp32
  int ldo;                       // output row stride (elements)
  const int32_t* rowroute;       // padded expert row -> route (or -1)
  const int2* tiles;             // (expert, first padded row) per M tile
  const int32_t* meta;           // [0] = number of M tiles
  const __nv_bfloat16* gatherA;  // MOE1: xn2 [T][512]
  float* ystage;                 // MOE2: [2T][512]
  int32_t* comb_cnt;             // MOE2: [T][2]
  const float* topk_w;           // MOE2: [T][2]
  int32_t* err;
};

enum { G_QKV = 0, G_OUT = 1, G_MOE1 = 2, G_MOE2 = 3 };

template <int BN>
struct GemmCfg {
  static constexpr int STAGES = BN >= 256 ? 4 : 6;
  static constexpr int A_BYTES = 128 * 64 * 2;
  static constexpr int B_BYTES = BN * 64 * 2;
  static constexpr int SMEM = STAGES * (A_BYTES + B_BYTES) + 1024 /*align*/ + 256 /*barriers*/;
};

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float (&v)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 u;
    u.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    u.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    u.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    u.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    d[q] = u;
  }
}
__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* src, float (&v)[32]) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 u = s[q];
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(p[i]);
      v[8 * q + 2 * i] = f.x;
      v[8 * q + 2 * i + 1] = f.y;
    }
  }
}

template <int BN, int MODE>
__global__ void __launch_bounds__(192, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmTcParams p) {
  using Cfg = GemmCfg<BN>;
  constexpr int STAGES = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * Cfg::B_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* accum = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  __shared__ int s_skip;
  __shared__ int2 s_tile;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    int skip = has_error(p.err) ? 1 : 0;
    int2 tl = make_int2(0, int(blockIdx.x) * 128);
    if (MODE >= G_MOE1) {
      if (int(blockIdx.x) >= p.meta[0]) skip = 1; else tl = p.tiles[blockIdx.x];
    }
    s_skip = skip;
    s_tile = tl;
    if (!skip) {
      for (int s = 0; s < STAGES; ++s) {
        mbar_init(&full[s], MODE == G_MOE1 ? 1 + 128 : 1);
        mbar_init(&empty[s], 1);
      }
      mbar_init(accum, 1);
      fence_mbar_init();
    }
  }
  __syncthreads();
  if (s_skip) return;
  const int expert = s_tile.x;
  const int m0 = s_tile.y;
  const int n0 = int(blockIdx.y) * BN;
  if (warp == 1) {
    tmem_alloc(tmem_slot, BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nkb = p.num_kb;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      const uint32_t tx = (MODE == G_MOE1 ? 0u : uint32_t(Cfg::A_BYTES)) + uint32_t(Cfg::B_BYTES);
      int issued = 0;
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % STAGES, round = kb / STAGES;
        if (round > 0 && !mbar_wait(&empty[s], (round - 1) & 1)) {
          set_error(p.err, PTL_ERR_TIMEOUT);
          break;
        }
        mbar_arrive_expect_tx(&full[s], tx);
        if (MODE != G_MOE1) tma_load_2d(sA + s * Cfg::A_BYTES, &tmA, &full[s], kb * 64, m0);
        tma_load_2d(sB + s * Cfg::B_BYTES, &tmB, &full[s], kb * 64, expert * p.N_total + n0);
        ++issued;
      }
      if (MODE != G_MOE1) {
        // Never leave with copies in flight: the last stages must have landed.
        for (int kb = issued > STAGES ? issued - STAGES : 0; kb < issued; ++kb)
          mbar_wait(&full[kb % STAGES], (kb / STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(128, BN);
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % STAGES, round = kb / STAGES;
        if (!mbar_wait(&full[s], round & 1)) {
          set_error(p.err, PTL_ERR_TIMEOUT);
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + s * Cfg::A_BYTES);
        const uint32_t b0 = smem_u32(sB + s * Cfg::B_BYTES);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16_ss(tmem, umma_desc_sw128(a0 + 32 * k, 1024), umma_desc_sw128(b0 + 32 * k, 1024),
                       idesc, (kb | k) != 0);
        umma_commit(&empty[s]);
      }
      umma_commit(accum);
    }
  } else {
    const int r = 32 * (warp & 3) + lane;  // accumulator row == TMEM lane
    if (MODE == G_MOE1) {
      // Gather producer: thread r fills row r of each A stage with the
      // 64-element K slice of its token's LayerNorm2 row, 16 bytes at a
      // time, at the 128-byte-swizzled position TMA would have used.
      const int route = p.rowroute[m0 + r];
      const __nv_bfloat16* src = route >= 0 ? p.gatherA + size_t(route >> 1) * D : nullptr;
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % STAGES, round = kb / STAGES;
        if (round > 0 && !mbar_wait(&empty[s], (round - 1) & 1)) {
          set_error(p.err, PTL_ERR_TIMEOUT);
          break;
        }
        uint4 v[8];
#pragma unroll
        for (int c = 0; c < 8; ++c)
          v[c] = src ? __ldg(reinterpret_cast<const uint4*>(src + kb * 64) + c) : make_uint4(0, 0, 0, 0);
        const uint32_t row_addr = smem_u32(sA + s * Cfg::A_BYTES) + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(row_addr + ((c ^ (r & 7)) << 4), v[c].x, v[c].y, v[c].z, v[c].w);
        fence_proxy_async_smem();
        mbar_arrive(&full[s]);
      }
    }
    const bool acc_ok = mbar_wait(accum, 0);
    if (!acc_ok) set_error(p.err, PTL_ERR_TIMEOUT);
    tc_fence_after();
    if (acc_ok) {
      const uint32_t taddr = tmem + (uint32_t(32 * (warp & 3)) << 16);
      const int row = m0 + r;
      if (MODE == G_MOE2) {
        const int route = p.rowroute[row];
        const int t = route >> 1;
#pragma unroll 1
        for (int j = 0; j < BN / 32; ++j) {
          uint32_t raw[32];
          tmem_ld32(taddr + 32 * j, raw);
          tmem_ld_wait();
          if (route >= 0) {
            const int n = n0 + 32 * j;
            const float* bb = p.bias ? p.bias + expert * p.N_total + n : nullptr;
            float4* dst = reinterpret_cast<float4*>(p.ystage + size_t(route) * D + n);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              float4 y;
              y.x = __uint_as_float(raw[4 * q + 0]) + (bb ? __ldg(bb + 4 * q + 0) : 0.f);
              y.y = __uint_as_float(raw[4 * q + 1]) + (bb ? __ldg(bb + 4 * q + 1) : 0.f);
              y.z = __uint_as_float(raw[4 * q + 2]) + (bb ? __ldg(bb + 4 * q + 2) : 0.f);
              y.w = __uint_as_float(raw[4 * q + 3]) + (bb ? __ldg(bb + 4 * q + 3) : 0.f);
              dst[q] = y;
            }
          }
        }
        if (route >= 0) {
          __threadfence();
          const int prev = atomicAdd(&p.comb_cnt[size_t(t) * GEMM2_NT + blockIdx.y], 1);
          if (prev == 1) {
            __threadfence();
            const float w0 = p.topk_w[2 * t], w1 = p.topk_w[2 * t + 1];
            const float* y0 = p.ystage + size_t(2 * t) * D;
            const float* y1 = p.ystage + size_t(2 * t + 1) * D;
#pragma unroll 1
            for (int j = 0; j < BN / 32; ++j) {
              const int n = n0 + 32 * j;
              float xr[32], o[32];
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 r4 = *(reinterpret_cast<const float4*>(p.resid_f32 + size_t(t) * D + n) + q);
                xr[4 * q + 0] = r4.x;
                xr[4 * q + 1] = r4.y;
                xr[4 * q + 2] = r4.z;
                xr[4 * q + 3] = r4.w;
              }
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 a = __ldcg(reinterpret_cast<const float4*>(y0 + n) + q);
                const float4 b = __ldcg(reinterpret_cast<const float4*>(y1 + n) + q);
                o[4 * q + 0] = (xr[4 * q + 0] + w0 * a.x) + w1 * b.x;
                o[4 * q + 1] = (xr[4 * q + 1] + w0 * a.y) + w1 * b.y;
                o[4 * q + 2] = (xr[4 * q + 2] + w0 * a.z) + w1 * b.z;
                o[4 * q + 3] = (xr[4 * q + 3] + w0 * a.w) + w1 * b.w;
              }
              store_bf16x32(p.out + size_t(t) * p.ldo + n, o);
            }
          }
        }
      } else {
#pragma unroll 1
        for (int j = 0; j < BN / 32; ++j) {
          uint32_t raw[32];
          tmem_ld32(taddr + 32 * j, raw);
          tmem_ld_wait();
          const int n = n0 + 32 * j;
          float v[32];
          const float* bb = p.bias ? p.bias + (MODE == G_MOE1 ? expert * p.N_total : 0) + n : nullptr;
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(raw[i]) + (bb ? __ldg(bb + i) : 0.f);
          if (MODE == G_MOE1) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = fmaxf(v[i], 0.f);
            store_bf16x32(p.out + size_t(row) * p.ldo + n, v);
          } else if (row < p.M) {
            if (MODE == G_OUT) {
              float xr[32];
              load_bf16x32(p.resid + size_t(row) * D + n, xr);
              float4* dst = reinterpret_cast<float4*>(p.out_f32 + size_t(row) * p.ldo + n);
#pragma unroll
              for (int q = 0; q < 8; ++q)
                dst[q] = make_float4(v[4 * q] + xr[4 * q], v[4 * q + 1] + xr[4 * q + 1],
                                     v[4 * q + 2] + xr[4 * q + 2], v[4 * q + 3] + xr[4 * q + 3]);
            } else {
              store_bf16x32(p.out + size_t(row) * p.ldo + n, v);
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

// ------------------------------------------------------------------ host
template <int BN, int MODE>
static int launch_one(const CUtensorMap& a, const CUtensorMap& b, const GemmTcParams& p, dim3 grid,
                      cudaStream_t st) {
  static bool configured = false;
  const int smem = GemmCfg<BN>::SMEM;
  if (!configured) {
    if (cudaFuncSetAttribute(gemm_tc_kernel<BN, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
      return -1;
    configured = true;
  }
  gemm_tc_kernel<BN, MODE><<<grid, 192, smem, st>>>(a, b, p);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -1;
}

int launch_gemm_qkv(const CUtensorMap& xn, const CUtensorMap& w, const float* bias, void* qkv, int T,
                    int32_t* err, cudaStream_t st) {
  GemmTcParams p{};
  p.M = T;
  p.N_total = QKV_N;
  p.num_kb = D / 64;
  p.bias = bias;
  p.out = static_cast<__nv_bfloat16*>(qkv);
  p.ldo = QKV_N;
  p.err = err;
  return launch_one<QKV_BN, G_QKV>(xn, w, p, dim3((T + 127) / 128, QKV_N / QKV_BN), st);
}

int launch_gemm_out(const CUtensorMap& attn, const CUtensorMap& w, const float* bias, const void* x,
                    void* x1, int T, int32_t* err, cudaStream_t st) {
  GemmTcParams p{};
  p.M = T;
  p.N_total = D;
  p.num_kb = D / 64;
  p.bias = bias;
  p.resid = static_cast<const __nv_bfloat16*>(x);
  p.out_f32 = static_cast<float*>(x1);
  p.ldo = D;
  p.err = err;
  return launch_one<OUT_BN, G_OUT>(attn, w, p, dim3((T + 127) / 128, D / OUT_BN), st);
}

int launch_gemm_moe1(const CUtensorMap& dummyA, const CUtensorMap& w1, const float* b1, const void* xn2,
                     const WsLayout& L, char* ws, cudaStream_t st) {
  GemmTcParams p{};
  p.N_total = F;
  p.num_kb = D / 64;
  p.bias = b1;
  p.out = reinterpret_cast<__nv_bfloat16*>(ws + L.hbuf);
  p.ldo = F;
  p.rowroute = reinterpret_cast<const int32_t*>(ws + L.rowroute);
  p.tiles = reinterpret_cast<const int2*>(ws + L.tiles);
  p.meta = reinterpret_cast<const int32_t*>(ws + L.route_meta);
  p.gatherA = static_cast<const __nv_bfloat16*>(xn2);
  p.err = reinterpret_cast<int32_t*>(ws + L.err);
  return launch_one<MOE1_BN, G_MOE1>(dummyA, w1, p, dim3(unsigned(L.max_tiles), F / MOE1_BN), st);
}

int launch_gemm_moe2(const CUtensorMap& hbuf, const CUtensorMap& w2, const float* b2, const void* x1,
                     const float* topk_w, void* out, const WsLayout& L, char* ws, cudaStream_t st) {
  GemmTcParams p{};
  p.N_total = D;
  p.num_kb = F / 64;
  p.bias = b2;
  p.resid_f32 = static_cast<const float*>(x1);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.ldo = D;
  p.rowroute = reinterpret_cast<const int32_t*>(ws + L.rowroute);
  p.tiles = reinterpret_cast<const int2*>(ws + L.tiles);
  p.meta = reinterpret_cast<const int32_t*>(ws + L.route_meta);
  p.ystage = reinterpret_cast<float*>(ws + L.ystage);
  p.comb_cnt = reinterpret_cast<int32_t*>(ws + L.comb_cnt);
  p.topk_w = topk_w;
  p.err = reinterpret_cast<int32_t*>(ws + L.err);
  return launch_one<GEMM2_BN, G_MOE2>(hbuf, w2, p, dim3(unsigned(L.max_tiles), D / GEMM2_BN), st);
}

}  // namespace ptl
